#!/usr/bin/env python
"""Benchmark of the B200 MoBA causal prefill forward pass.

`python bench.py --gpus N --steps K --warmup W [--config 1m]` prints one JSON
line. A step is one whole forward pass (pool, gate, router, attention, merge)
over one synthetic sequence resident in HBM. The default workload is the
1M-token one (32 q / 8 kv heads, block 4096, top-12): the largest single-GPU
configuration, with the most work of the five. With N > 1 (launched by
torch.distributed.run) every rank runs its own independent sequence: weak
scaling, no collective on the data path (a MAX all-reduce of the timings
only).

`--impl reference` times the fp64 CPU oracle instead (on rank 0), on a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth_inputs as si  # noqa: E402

METRIC = "MoBA prefill tokens/s and effective TFLOP/s (selected blocks) vs bf16 TC roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLUSH_BYTES = 256 << 20  # twice the 126 MB L2


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def tensor_peak(peaks, peaks_src, ms_per_step):
    """bf16 dense peak for a kernel timed inside a step: the burst figure for
    steps under 200 ms, the sustained (power-capped) one for longer steps."""
    long_step = ms_per_step > 200.0
    key = "bf16_tflops_sustained" if long_step else "bf16_tflops"
    return peaks[key], f"{peaks_src} bf16 {'sustained' if long_step else 'burst'}"


def attn_traffic(workload_name: str):
    """DRAM bytes of the attention kernel per step (its launches summed) from
    the committed ncu record, or None when the record is for another workload
    or an older attention kernel."""
    import hashlib
    rec = os.path.join(ROOT, "profiles", "attn_kernel_traffic.txt")
    src = os.path.join(ROOT, "block_sparse_long_fwd_b200", "csrc", "attn.cuh")
    try:
        kv = {}
        for line in open(rec):
            if "=" in line and not line.lstrip().startswith("#"):
                k, v = line.split("=", 1)
                kv[k.strip()] = v.strip()
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
        if kv.get("kernel_source_sha256") == sha and kv.get("workload") == workload_name:
            return int(kv["bytes_per_step"])
    except (OSError, ValueError, KeyError):
        pass
    return None


def routed_rows(w) -> int:
    """Past-block partials per step: sum over rows of min(k-1, t//B)."""
    nb = w.nblocks
    k_eff = min(w.topk, nb)
    tot = 0
    for b in range(nb):
        n = min(w.seqlen, (b + 1) * w.block_size) - b * w.block_size
        tot += n * min(k_eff - 1, b)
    return tot * w.heads_q


def stage_bytes(w) -> dict:
    """Algorithmic HBM bytes per step of the memory-bound stages."""
    d = w.head_dim
    k_eff = min(w.topk, w.nblocks)
    nbp = max(w.nblocks - 1, 0)
    r = routed_rows(w)
    if w.nblocks > 1 and k_eff == w.nblocks:
        # full causal attention runs as one causal pass: no means, no scores,
        # one selection entry and one partial per row
        rows = w.seqlen * w.heads_q
        return {"pool": 0, "gate": rows * 4, "merge": rows * 4 + 2 * rows * (d * 2 + 4)}
    return {
        # read every key that can be pooled once, write the means
        "pool": nbp * w.block_size * w.heads_kv * d * 2 + nbp * w.heads_kv * d * 4,
        # read Q once and the means, write the selection table
        "gate": w.seqlen * w.heads_q * d * 2 + nbp * w.heads_kv * d * 4 + w.seqlen * w.heads_q * k_eff * 4,
        # read the table and every partial (O fp16 + lse), write out bf16 + lse
        "merge": w.seqlen * w.heads_q * k_eff * 4 + (r + w.seqlen * w.heads_q) * (d * 2 + 4)
        + w.seqlen * w.heads_q * (d * 2 + 4),
    }


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_uuid: str | None):
        self.proc = None
        self.lines = []
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if device_uuid:
            cmd += ["-i", device_uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def replica_workload(w, rank: int):
    """Rank r's own sequence: the workload's shape, an independent seed."""
    return si.Workload(w.name, w.seqlen, w.heads_q, w.heads_kv, w.head_dim, w.block_size, w.topk,
                       w.seed + 7919 * rank)


def max_over_ranks(values, device, world: int):
    """Element-wise MAX of per-rank timings (every rank takes this step)."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_tokens_per_s(world: int, seqlen: int, steps: int, max_total_ms: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return world * seqlen * steps / (max_total_ms / 1e3)


# ------------------------------------------------------------------ oracle

def oracle_sample(w, seconds: float, seed: int):
    """Time the fp64 oracle on a seeded sample of rows of workload w.

    Returns (tokens/s, threads, description). Per-token cost = pool cost / S +
    (gate + attention cost of one row) * heads_q.
    """
    import oracle
    threads = oracle.threads()
    rng = np.random.default_rng(seed)
    q = np.empty((w.seqlen, w.heads_q, w.head_dim), dtype=np.uint16)
    k = np.empty((w.seqlen, w.heads_kv, w.head_dim), dtype=np.uint16)
    v = np.empty((w.seqlen, w.heads_kv, w.head_dim), dtype=np.uint16)
    si.fill_q(q.ctypes.data, w)
    si.fill_k(k.ctypes.data, w)
    si.fill_v(v.ctypes.data, w)
    t0 = time.perf_counter()
    m = oracle.kmean(k, w.block_size)
    t_pool = time.perf_counter() - t0

    def run(n):
        rt = rng.integers(0, w.seqlen, size=n).astype(np.int64)
        rh = rng.integers(0, w.heads_q, size=n).astype(np.int32)
        s = time.perf_counter()
        oracle.attend(q, k, v, w.block_size, w.topk, rt, rh, m=m, nthreads=threads)
        return time.perf_counter() - s

    n = max(threads, 8)
    dt = run(n)
    while dt < 0.5 and n < (1 << 22):
        n *= 4
        dt = run(n)
    n_final = max(n, int(n * max(seconds - t_pool, 0.5) / max(dt, 1e-9)))
    return q, k, v, m, t_pool, run, n_final, threads


def run_reference(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    per_step = 2.0
    q, k, v, m, t_pool, run, n, threads = oracle_sample(w, per_step, w.seed + 4242)
    for _ in range(args.warmup):
        run(max(n // 8, 1))
    times = [run(n) for _ in range(args.steps)]
    t_row = statistics.mean(times) / n
    tok_s = 1.0 / (t_pool / w.seqlen + t_row * w.heads_q)
    line = {
        "impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * w.seqlen / tok_s,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args.gpus),
        "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{n} uniformly drawn (token, head) rows per step, gate + masked softmax in fp64; "
                                   f"full-sequence key mean-pool timed once ({t_pool:.2f} s) and amortised over "
                                   f"{w.seqlen} tokens"},
        "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def chunk_flops(w, q0: int) -> float:
    """Selected-block FLOPs of the rows q0..S-1 (4*d*Hq per unmasked pair)."""
    B, S = w.block_size, w.seqlen
    k_eff = min(w.topk, w.nblocks)
    t = np.arange(q0, S, dtype=np.int64)
    b = t // B
    keys = np.where(k_eff >= w.nblocks, t + 1, np.minimum(k_eff - 1, b) * B + (t % B) + 1)
    return 4.0 * w.head_dim * w.heads_q * float(keys.sum())


DECODE_ROWS = 64  # chunks of at most this many query tokens are reported against HBM


def chunk_kv_bytes(w, q_h, k, q0: int) -> int:
    """Algorithmic HBM bytes of the attention for the queries of tokens
    q0..S-1: per kv head, the K and V rows of every block that some of its q
    heads' rows attend (own block up to the last query token, plus the past
    blocks the gate picks), the chunk's Q rows and its partial outputs. The
    picks are recomputed here from the library's pooled block means (a
    measurement helper: which blocks are read, not how they are combined)."""
    import torch

    import block_sparse_long_fwd_b200 as moba
    S, B, d = w.seqlen, w.block_size, w.head_dim
    G = w.heads_q // w.heads_kv
    P = min(w.topk, w.nblocks) - 1
    km = moba.pool(k, B).double().cpu().numpy()  # [Hkv][nbp][d]
    q = q_h[q0:].view(torch.int16).numpy().astype(np.uint32) << 16
    q = q.view(np.float32).astype(np.float64)  # [n][Hq][d]
    keys = 0  # K/V rows read, summed over kv heads
    own_last = {}  # own block -> its last token with a query
    for t in range(q0, S):
        own_last[t // B] = t
    for g in range(w.heads_kv):
        past = set()
        for tl in range(S - q0):
            t = q0 + tl
            b = t // B
            if b and P:
                s = q[tl, g * G:(g + 1) * G] @ km[g, :b].T  # [G][b]
                for row in s:
                    past.update(np.argsort(-row, kind="stable")[:P].tolist())
        past -= set(own_last)
        keys += len(past) * B + sum(t - b * B + 1 for b, t in own_last.items())
    rows = (S - q0) * w.heads_q
    return int(keys * d * 2 * 2 + rows * d * 2 + rows * min(w.topk, w.nblocks) * (d * 2 + 4))


def run_chunk(args, w):
    """--chunk N: the last N tokens' queries against the whole cache
    (moba_fwd_chunk; N = 1 is one decode step). One GPU."""
    import torch

    import block_sparse_long_fwd_b200 as moba

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    S, Hq, Hkv, d = w.seqlen, w.heads_q, w.heads_kv, w.head_dim
    n = args.chunk
    q0 = S - n
    q_h = torch.empty((S, Hq, d), dtype=torch.bfloat16, pin_memory=True)
    k_h = torch.empty((S, Hkv, d), dtype=torch.bfloat16, pin_memory=True)
    v_h = torch.empty((S, Hkv, d), dtype=torch.bfloat16, pin_memory=True)
    si.fill_q(q_h.data_ptr(), w)
    si.fill_k(k_h.data_ptr(), w)
    si.fill_v(v_h.data_ptr(), w)
    qc = q_h[q0:].to(dev)
    k, v = k_h.to(dev), v_h.to(dev)
    out = torch.empty((n, Hq, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((Hq, n), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    # --cached-means: block means pooled once, outside the timed steps (a
    # decode loop pools again only when the cache completes a block)
    kmean = moba.pool(k, w.block_size) if args.cached_means else None
    for _ in range(args.warmup):
        flush.zero_()
        moba.fwd_chunk(qc, k, v, w.block_size, w.topk, out=out, lse=lse, kmean=kmean)
    sampler = ClockSampler(None)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        moba.fwd_chunk(qc, k, v, w.block_size, w.topk, out=out, lse=lse, kmean=kmean)
        b.record(stream)
    torch.cuda.synchronize()
    total_ms = sum(a.elapsed_time(b) for a, b in ev)
    moba.profile_begin()
    for _ in range(args.steps):
        flush.zero_()
        moba.fwd_chunk(qc, k, v, w.block_size, w.topk, out=out, lse=lse, kmean=kmean)
    stages, launches, calls = moba.profile_end()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if moba.device_status() != 0:
        raise RuntimeError("device status set: " + moba.last_error())
    # end to end: each step uploads the chunk's new q, k, v rows into the
    # resident cache, runs the chunk and reads out and lse back
    out_h = torch.empty((n, Hq, d), dtype=torch.bfloat16, pin_memory=True)
    lse_h = torch.empty((Hq, n), dtype=torch.float32, pin_memory=True)
    e2e_steps = max(1, min(args.steps, 10))
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        qc.copy_(q_h[q0:], non_blocking=True)
        k[q0:].copy_(k_h[q0:], non_blocking=True)
        v[q0:].copy_(v_h[q0:], non_blocking=True)
        moba.fwd_chunk(qc, k, v, w.block_size, w.topk, out=out, lse=lse, kmean=kmean)
        out_h.copy_(out, non_blocking=True)
        lse_h.copy_(lse, non_blocking=True)
        torch.cuda.synchronize()
    e2e_ms = 1e3 * (time.perf_counter() - t0)
    peaks, peaks_src = load_peaks()
    flops = chunk_flops(w, q0)
    attn_ms = stages["attention"] / max(calls, 1)
    achieved = flops / (attn_ms / 1e3) / 1e12
    if n <= DECODE_ROWS:
        # a few query tokens: the attention streams the K/V rows of the blocks
        # they attend, so it is bound by HBM, not by the tensor cores
        kv_bytes = chunk_kv_bytes(w, q_h, k, q0)
        gbs = kv_bytes / (attn_ms / 1e3) / 1e9
        roofline = {"bound": "hbm", "kernel": "attn_kernel", "achieved": gbs, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                    "peak_source": f"{peaks_src} HBM copy",
                    "algorithmic": f"{kv_bytes:.4e} bytes: K and V rows of the distinct blocks the chunk's rows attend "
                                   "(per kv head), its Q rows and its partial outputs / attention ms",
                    "tflops": achieved}
    else:
        peak, psrc = tensor_peak(peaks, peaks_src, total_ms / args.steps)
        roofline = {"bound": "tensor", "kernel": "attn_kernel", "achieved": achieved,
                    "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                    "traffic": None, "peak_source": psrc,
                    "algorithmic": f"{flops:.4e} selected-block FLOPs of the chunk's rows / attention ms"}
    line = {
        "metric": METRIC, "value": n * args.steps / (total_ms / 1e3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(w, 1), mode="decode" if n == 1 else "chunked prefill", q_start=q0, chunk=n,
                       block_means="cached (pooled once)" if args.cached_means else "pooled every call"),
        "eff_tflops": flops * args.steps / (total_ms / 1e3) / 1e12,
        "stage_ms_per_step": {kk: vv / max(calls, 1) for kk, vv in stages.items() if not kk.startswith("bwd_")},
        "roofline": roofline,
        "e2e": {"value": n * e2e_steps / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(n * (Hq + 2 * Hkv) * d * 2),
                "d2h_bytes_per_step": int(out_h.nbytes + lse_h.nbytes)},
        "gpu_launches": launches // max(calls, 1) * args.steps,
        "gpu_launches_per_step": launches / max(calls, 1),
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_backward(args, w):
    """--backward: the gradient (moba_bwd) of the workload's forward pass,
    given its out and lse; one GPU. FLOPs: the five products of attention's
    gradient per attended pair (S recomputed, dP, dV, dK, dQ: 2.5 times the
    forward's), plus dP and S recomputed once more in the dQ kernel."""
    import torch

    import block_sparse_long_fwd_b200 as moba

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    S, Hq, Hkv, d = w.seqlen, w.heads_q, w.heads_kv, w.head_dim
    q_h = torch.empty((S, Hq, d), dtype=torch.bfloat16, pin_memory=True)
    k_h = torch.empty((S, Hkv, d), dtype=torch.bfloat16, pin_memory=True)
    v_h = torch.empty((S, Hkv, d), dtype=torch.bfloat16, pin_memory=True)
    do_h = torch.empty((S, Hq, d), dtype=torch.bfloat16, pin_memory=True)
    si.fill_q(q_h.data_ptr(), w)
    si.fill_k(k_h.data_ptr(), w)
    si.fill_v(v_h.data_ptr(), w)
    si.fill_dout(do_h.data_ptr(), w)
    q, k, v, do = q_h.to(dev), k_h.to(dev), v_h.to(dev), do_h.to(dev)
    out, lse = moba.fwd(q, k, v, w.block_size, w.topk)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        flush.zero_()
        moba.bwd(q, k, v, out, lse, do, w.block_size, w.topk)
    sampler = ClockSampler(None)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        moba.bwd(q, k, v, out, lse, do, w.block_size, w.topk)
        b.record(stream)
    torch.cuda.synchronize()
    total_ms = sum(a.elapsed_time(b) for a, b in ev)
    moba.profile_begin()
    for _ in range(args.steps):
        flush.zero_()
        moba.bwd(q, k, v, out, lse, do, w.block_size, w.topk)
    stages, launches, calls = moba.profile_end()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if moba.device_status() != 0:
        raise RuntimeError("device status set: " + moba.last_error())
    # end to end: upload q, k, v, out, lse, dO; read dq, dk, dv back
    out_h, lse_h = out.cpu().pin_memory(), lse.cpu().pin_memory()
    dq_h = torch.empty((S, Hq, d), dtype=torch.bfloat16, pin_memory=True)
    dk_h = torch.empty((S, Hkv, d), dtype=torch.bfloat16, pin_memory=True)
    dv_h = torch.empty((S, Hkv, d), dtype=torch.bfloat16, pin_memory=True)
    e2e_steps = max(1, min(args.steps, 5))
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        for dst, src in ((q, q_h), (k, k_h), (v, v_h), (out, out_h), (lse, lse_h), (do, do_h)):
            dst.copy_(src, non_blocking=True)
        dq, dk, dv = moba.bwd(q, k, v, out, lse, do, w.block_size, w.topk)
        dq_h.copy_(dq, non_blocking=True)
        dk_h.copy_(dk, non_blocking=True)
        dv_h.copy_(dv, non_blocking=True)
        torch.cuda.synchronize()
    e2e_ms = 1e3 * (time.perf_counter() - t0)
    peaks, peaks_src = load_peaks()
    fwd_flops = chunk_flops(w, 0)
    per = {kk: vv / max(calls, 1) for kk, vv in stages.items() if kk not in ("attention", "merge")}
    dkdv_flops = 2.0 * fwd_flops  # S^T, dP^T, dV, dK
    peak, psrc = tensor_peak(peaks, peaks_src, total_ms / args.steps)
    achieved = dkdv_flops / (per["bwd_dkdv"] / 1e3) / 1e12
    line = {
        "metric": METRIC, "value": S * args.steps / (total_ms / 1e3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(w, 1), mode="backward (dq, dk, dv given out, lse, dout)"),
        "eff_tflops": 2.5 * fwd_flops * args.steps / (total_ms / 1e3) / 1e12,
        "stage_ms_per_step": per,
        "roofline": {"bound": "tensor", "kernel": "bwd_dkdv_kernel", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": None, "peak_source": psrc,
                     "algorithmic": f"{dkdv_flops:.4e} FLOPs (S^T, dP^T, dV, dK per attended pair) / dK-dV ms",
                     "dq_kernel_tflops": 1.5 * fwd_flops / (per["bwd_dq"] / 1e3) / 1e12},
        "e2e": {"value": S * e2e_steps / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(q_h.nbytes + k_h.nbytes + v_h.nbytes + out_h.nbytes + lse_h.nbytes
                                          + do_h.nbytes),
                "d2h_bytes_per_step": int(dq_h.nbytes + dk_h.nbytes + dv_h.nbytes)},
        "gpu_launches": launches // max(calls, 1) * args.steps,
        "gpu_launches_per_step": launches / max(calls, 1),
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def varlen_lengths(w, n: int):
    """--varlen N: the workload's tokens cut into N sequences at seeded
    uniform cut points (each at least 1 token)."""
    rng = np.random.default_rng(w.seed + 7919)
    cuts = np.sort(rng.choice(np.arange(1, w.seqlen), size=n - 1, replace=False)) if n > 1 else np.array([], int)
    edges = np.concatenate([[0], cuts, [w.seqlen]]).astype(np.int64)
    return np.diff(edges), edges


def run_varlen(args, w):
    """--varlen N: one packed batch of N independent sequences of the
    workload's head shape, block size and top-k (moba_fwd_varlen). One GPU."""
    import torch

    import block_sparse_long_fwd_b200 as moba

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    T, Hq, Hkv, d = w.seqlen, w.heads_q, w.heads_kv, w.head_dim
    lengths, cu = varlen_lengths(w, args.varlen)
    subs = [si.Workload(f"{w.name}_seq{b}", int(L), Hq, Hkv, d, w.block_size, w.topk, w.seed + 1000 + b)
            for b, L in enumerate(lengths)]
    q_h = torch.empty((T, Hq, d), dtype=torch.bfloat16, pin_memory=True)
    k_h = torch.empty((T, Hkv, d), dtype=torch.bfloat16, pin_memory=True)
    v_h = torch.empty((T, Hkv, d), dtype=torch.bfloat16, pin_memory=True)
    for b, sw in enumerate(subs):
        a, e = int(cu[b]), int(cu[b + 1])
        si.fill_q(q_h[a:e].data_ptr(), sw)
        si.fill_k(k_h[a:e].data_ptr(), sw)
        si.fill_v(v_h[a:e].data_ptr(), sw)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    out = torch.empty((T, Hq, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((Hq, T), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        flush.zero_()
        moba.fwd_varlen(q, k, v, cu, w.block_size, w.topk, out=out, lse=lse)
    sampler = ClockSampler(None)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        moba.fwd_varlen(q, k, v, cu, w.block_size, w.topk, out=out, lse=lse)
        b.record(stream)
    torch.cuda.synchronize()
    total_ms = sum(a.elapsed_time(b) for a, b in ev)
    moba.profile_begin()
    for _ in range(args.steps):
        flush.zero_()
        moba.fwd_varlen(q, k, v, cu, w.block_size, w.topk, out=out, lse=lse)
    stages, launches, calls = moba.profile_end()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if moba.device_status() != 0:
        raise RuntimeError("device status set: " + moba.last_error())
    out_h = torch.empty((T, Hq, d), dtype=torch.bfloat16, pin_memory=True)
    lse_h = torch.empty((Hq, T), dtype=torch.float32, pin_memory=True)
    e2e_steps = max(1, min(args.steps, 5))
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        q.copy_(q_h, non_blocking=True)
        k.copy_(k_h, non_blocking=True)
        v.copy_(v_h, non_blocking=True)
        moba.fwd_varlen(q, k, v, cu, w.block_size, w.topk, out=out, lse=lse)
        out_h.copy_(out, non_blocking=True)
        lse_h.copy_(lse, non_blocking=True)
        torch.cuda.synchronize()
    e2e_ms = 1e3 * (time.perf_counter() - t0)
    peaks, peaks_src = load_peaks()
    flops = sum(chunk_flops(sw, 0) for sw in subs)
    attn_ms = stages["attention"] / args.steps
    achieved = flops / (attn_ms / 1e3) / 1e12
    peak, psrc = tensor_peak(peaks, peaks_src, total_ms / args.steps)
    line = {
        "metric": METRIC, "value": T * args.steps / (total_ms / 1e3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(w, 1), mode="packed batch", batch_per_gpu=int(args.varlen),
                       lengths=[int(x) for x in lengths]),
        "eff_tflops": flops * args.steps / (total_ms / 1e3) / 1e12,
        "stage_ms_per_step": {kk: vv / args.steps for kk, vv in stages.items() if not kk.startswith("bwd_")},
        "roofline": {"bound": "tensor", "kernel": "attn_kernel", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": None, "peak_source": psrc,
                     "algorithmic": f"{flops:.4e} selected-block FLOPs of all sequences / attention ms"},
        "e2e": {"value": T * e2e_steps / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(q_h.nbytes + k_h.nbytes + v_h.nbytes),
                "d2h_bytes_per_step": int(out_h.nbytes + lse_h.nbytes)},
        "gpu_launches": launches // args.steps * args.steps,
        "gpu_launches_per_step": launches / args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, n):
    return {"workload": w.name, "seqlen": w.seqlen, "heads_q": w.heads_q, "heads_kv": w.heads_kv,
            "head_dim": w.head_dim, "block_size": w.block_size, "topk": w.topk, "batch_per_gpu": 1,
            "global_batch": n, "parallelism": f"replicas{n}" if n > 1 else "single",
            "l2": f"flushed between timed steps ({FLUSH_BYTES >> 20} MiB write)"}


# --------------------------------------------------------------------- ours

def run_ours(args, w):
    import torch
    import torch.distributed as dist

    import block_sparse_long_fwd_b200 as moba

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    # every rank: its own sequence (independent seed), same shape
    wr = replica_workload(w, rank)
    S, Hq, Hkv, d = wr.seqlen, wr.heads_q, wr.heads_kv, wr.head_dim
    q_h = torch.empty((S, Hq, d), dtype=torch.bfloat16, pin_memory=True)
    k_h = torch.empty((S, Hkv, d), dtype=torch.bfloat16, pin_memory=True)
    v_h = torch.empty((S, Hkv, d), dtype=torch.bfloat16, pin_memory=True)
    si.fill_q(q_h.data_ptr(), wr)
    si.fill_k(k_h.data_ptr(), wr)
    si.fill_v(v_h.data_ptr(), wr)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((Hq, S), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        flush.zero_()
        moba.fwd(q, k, v, wr.block_size, wr.topk, out=out, lse=lse)
    if moba.device_status() != 0:
        raise RuntimeError("device status set during warm-up: " + moba.last_error())

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:  # noqa: BLE001
        uuid = None
    sampler = ClockSampler(uuid)
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    # timed region 1 (the value): the calls a user makes; after the second
    # call with the same buffers the library replays a CUDA graph
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        moba.fwd(q, k, v, wr.block_size, wr.topk, out=out, lse=lse)
        ends[i].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    # timed region 2 (per-stage breakdown and the attention kernel's own
    # duration for the roofline): the same steps with the library's stage
    # events, launched kernel by kernel
    prof_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    prof_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    moba.profile_begin()
    for i in range(args.steps):
        flush.zero_()
        prof_s[i].record(stream)
        moba.fwd(q, k, v, wr.block_size, wr.topk, out=out, lse=lse)
        prof_e[i].record(stream)
    stages, launches, calls = moba.profile_end()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    prof_ms = sum(s_.elapsed_time(e_) for s_, e_ in zip(prof_s, prof_e)) / args.steps
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = sum(step_ms)
    # keep the GPU busy for >= 1 s so the clock samples see the load
    t_pad = time.perf_counter()
    while not args.no_pad and time.perf_counter() - t_pad < max(0.0, 1.0 - total_ms / 1e3):
        moba.fwd(q, k, v, wr.block_size, wr.topk, out=out, lse=lse)
        torch.cuda.synchronize()
    clocks = sampler.stop()
    status = moba.device_status()
    if status != 0:
        raise RuntimeError("device status set during timing: " + moba.last_error())

    # end to end through the public API: host buffers in, host buffers out
    out_h = torch.empty((S, Hq, d), dtype=torch.bfloat16, pin_memory=True)
    lse_h = torch.empty((Hq, S), dtype=torch.float32, pin_memory=True)
    e2e_steps = max(1, min(args.steps, 10))
    moba.fwd_host(q_h, k_h, v_h, wr.block_size, wr.topk, out=out_h, lse=lse_h)
    if world > 1:
        dist.barrier()
    e2e_ms = []
    for _ in range(e2e_steps):
        t0 = time.perf_counter()
        moba.fwd_host(q_h, k_h, v_h, wr.block_size, wr.topk, out=out_h, lse=lse_h)
        e2e_ms.append(1e3 * (time.perf_counter() - t0))
    e2e_total = sum(e2e_ms)

    # max over ranks of the device time
    total_ms, e2e_total, _ = max_over_ranks([total_ms, e2e_total, stages["attention"]], dev, world)

    line = None
    if rank == 0:
        peaks, peaks_src = load_peaks()
        flops = moba.effective_flops(S, Hq, wr.block_size, wr.topk, d)
        value = job_tokens_per_s(world, S, args.steps, total_ms)
        ms_per_step = total_ms / args.steps
        attn_ms = stages["attention"] / max(calls, 1)
        peak, psrc = tensor_peak(peaks, peaks_src, ms_per_step)
        achieved = flops / (attn_ms / 1e3) / 1e12
        sb = stage_bytes(wr)
        stage_roof = {}
        for st in ("pool", "gate", "merge"):
            ms = stages[st] / max(calls, 1)
            if ms > 0:
                gbs = sb[st] / (ms / 1e3) / 1e9
                stage_roof[st] = {"ms": ms, "bytes": sb[st], "gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"]}
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(wr, world),
            "eff_tflops": world * flops * args.steps / (total_ms / 1e3) / 1e12,
            "stage_ms_per_step": {kk: vv / max(calls, 1) for kk, vv in stages.items() if not kk.startswith("bwd_")},
            "ms_per_step_kernel_by_kernel": prof_ms,
            "roofline": {"bound": "tensor", "kernel": "attn_kernel", "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak, "traffic": attn_traffic(wr.name),
                         "peak_source": psrc,
                         "algorithmic": f"{flops:.4e} selected-block FLOPs per step / attention ms per step"},
            "stage_roofline_hbm": stage_roof,
            "e2e": {"value": job_tokens_per_s(world, S, e2e_steps, e2e_total), "unit": "tokens/s",
                    "h2d_bytes_per_step": int(q_h.nbytes + k_h.nbytes + v_h.nbytes),
                    "d2h_bytes_per_step": int(out_h.nbytes + lse_h.nbytes)},
            "gpu_launches": launches // max(calls, 1) * args.steps,
            "gpu_launches_per_step": launches / max(calls, 1),
            "gpu_launches_note": "kernels of ours per step, counted by the library in the breakdown loop; the value "
                                 "loop runs the same kernels replayed from a CUDA graph",
            "clocks": clocks,
            "clocks_window": "timed region, padded with untimed steps to >= 1 s",
        }
        if world == 1 and not args.no_cpu_baseline:
            q_, k_, v_, m_, t_pool, run, n, threads = oracle_sample(wr, args.cpu_seconds, wr.seed + 4242)
            dt = run(n)
            tok_s = 1.0 / (t_pool / S + dt / n * Hq)
            line["cpu_baseline"] = {
                "value": tok_s, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                "sample": f"{n} uniformly drawn (token, head) rows, gate + masked softmax in fp64 ({dt:.1f} s); "
                          f"full-sequence key mean-pool timed once ({t_pool:.2f} s) and amortised over {S} tokens"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", choices=sorted(si.WORKLOADS), default="1m")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--seqlen", type=int, default=0, help="override the workload's seqlen (profiling cases)")
    ap.add_argument("--heads", type=str, default="",
                    help="override the workload's q:kv heads, e.g. 4:1 (profiling cases)")
    ap.add_argument("--no-pad", action="store_true", help="no untimed load after the timed steps (profiling)")
    ap.add_argument("--chunk", type=int, default=0,
                    help="time only the last N tokens' queries against the whole cache (1 = one decode step)")
    ap.add_argument("--cached-means", action="store_true",
                    help="with --chunk: pool the block means once instead of on every call")
    ap.add_argument("--varlen", type=int, default=0,
                    help="time one packed batch of N independent sequences that together hold the workload's tokens")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (moba_bwd) of the workload instead of the forward")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = si.WORKLOADS[args.config]
    if args.seqlen:
        w = si.Workload(f"{w.name}_s{args.seqlen}", args.seqlen, w.heads_q, w.heads_kv, w.head_dim, w.block_size,
                        w.topk, w.seed)
    if args.heads:
        try:
            hq, hkv = (int(x) for x in args.heads.split(":"))
        except ValueError:
            ap.error("--heads takes q:kv, e.g. 4:1")
        if hq < 1 or hkv < 1 or hq % hkv:
            ap.error("--heads: q heads must be a positive multiple of kv heads")
        w = si.Workload(f"{w.name}_h{hq}kv{hkv}", w.seqlen, hq, hkv, w.head_dim, w.block_size, w.topk, w.seed)
    # one timed mode at a time, checked before any GPU work
    if sum(bool(x) for x in (args.chunk, args.varlen, args.backward)) > 1:
        ap.error("--chunk, --varlen and --backward are separate modes: give at most one")
    if args.cached_means and not args.chunk:
        ap.error("--cached-means applies to --chunk")
    if args.chunk and not 1 <= args.chunk <= w.seqlen:
        ap.error("--chunk must be in [1, seqlen]")
    if args.varlen and not 1 <= args.varlen <= w.seqlen:
        ap.error("--varlen must be in [1, seqlen]")
    if args.impl == "reference":
        return run_reference(args, w)
    if args.chunk:
        return run_chunk(args, w)
    if args.backward:
        return run_backward(args, w)
    if args.varlen:
        return run_varlen(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
