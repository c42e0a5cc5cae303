"""Shared helpers for the GPU-vs-oracle parity tests (test infrastructure).

Tolerances (bf16 inputs, fp32 accumulation, fp64 oracle):
  out: max-abs <= 2e-2 and mean-abs <= 2e-3; lse: abs <= 1e-3;
  selected block sets bit-exact wherever the oracle's gap between the last
  chosen and the first left-out past score exceeds 1e-3 of the row's largest
  |gate score| (its scale); below that, a GPU set is accepted when every
  chosen block scores at least the oracle's cut minus 1e-3 of that scale,
  and the oracle then recomputes that row with the GPU's set for the output
  comparison. (Relative to the two cut scores alone, the gap's denominator
  vanishes as they approach zero: on the 128K workload, row t=117994 h=23
  has cut scores -0.010217 and -0.010253, 0.35 % apart but 3.6e-5 apart in
  absolute terms, below what an fp32 evaluation of the 128-term inner
  products can order; against the row's largest score, 17.4, the gap is
  2e-6.)
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth_inputs as si

OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
LSE_ABS = 1e-3
GAP_REL = 1e-3


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()


def bf16_bits(x) -> np.ndarray:
    """fp32 values rounded to nearest-even bf16, as uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def make_inputs(S, Hq, Hkv, B, topk, seed):
    w = si.Workload("case", S, Hq, Hkv, 128, B, topk, seed)
    q, k, v = si.make_qkv(w)
    return w, q, k, v


def check_selection(q, k, sel_gpu_rows, rows_t, rows_h, B, Hkv, topk, m=None):
    """sel_gpu_rows [n][k_eff] int32 for rows (rows_t, rows_h). Returns the
    accepted selection (the GPU's) after checking it against the oracle."""
    m = oracle.kmean(k, B) if m is None else m
    sel_o, info = oracle.select(q, m, B, Hkv, topk, rows_t, rows_h)
    assert sel_gpu_rows.shape == sel_o.shape
    diff = np.any(sel_gpu_rows != sel_o, axis=1)
    if diff.any():
        bad = np.nonzero(diff)[0]
        for r in bad:
            gap, cut, scale = info[r, 0], info[r, 1], info[r, 3]
            assert gap <= GAP_REL, (
                f"row t={rows_t[r]} h={rows_h[r]}: gpu {sel_gpu_rows[r]} oracle {sel_o[r]} gap {gap}")
            t, h = int(rows_t[r]), int(rows_h[r])
            s = oracle.gate_scores(q, m, B, Hkv, t, h)
            chosen = [j for j in sel_gpu_rows[r] if 0 <= j < t // B]
            assert len(chosen) == len([j for j in sel_o[r] if 0 <= j < t // B])
            assert all(s[j] >= cut - GAP_REL * scale for j in chosen)
    return sel_gpu_rows, int(diff.sum())


def compare_outputs(out_gpu_rows, lse_gpu_rows, out_o, lse_o):
    """out_gpu_rows [n][128] float (from bf16), lse [n]; oracle fp64."""
    err = np.abs(out_gpu_rows.astype(np.float64) - out_o)
    lerr = np.abs(lse_gpu_rows.astype(np.float64) - lse_o)
    stats = dict(out_max=float(err.max()), out_mean=float(err.mean()), lse_max=float(lerr.max()))
    assert stats["out_max"] <= OUT_MAX_ABS, stats
    assert stats["out_mean"] <= OUT_MEAN_ABS, stats
    assert stats["lse_max"] <= LSE_ABS, stats
    return stats


def run_gpu(q, k, v, B, topk):
    import block_sparse_long_fwd_b200 as moba
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    out, lse = moba.fwd(qd, kd, vd, B, topk)
    kmean = moba.pool(kd, B)
    Hkv = k.shape[1]
    sel = moba.gate(qd, kmean, Hkv, B, topk)
    assert moba.device_status() == 0
    torch.cuda.synchronize()
    # out stays bf16 on the host (the 1M workload's output is 8.6 GB as bf16)
    return (out.cpu(), lse.cpu().numpy(), sel.cpu().numpy(), kmean.cpu().numpy())


def check_sel_structure(sel, S, B, topk):
    """Every GPU row: ascending distinct past blocks, own block last, -1 pad."""
    Hq, S_, k_eff = sel.shape
    assert S_ == S
    t = np.arange(S)
    bt = t // B
    npast = np.minimum(k_eff - 1, bt)
    for h in range(Hq):
        s = sel[h]
        own = s[t, npast]
        assert np.array_equal(own, bt)
        col = np.arange(k_eff)[None, :]
        past = np.where(col < npast[:, None], s, -2)
        assert np.all((past == -2) | ((past >= 0) & (past < bt[:, None])))
        if k_eff > 2:
            inc = np.diff(s, axis=1)
            inner = col[:, 1:] < npast[:, None]
            assert np.all(inc[inner] > 0)
        pad = np.where(col > npast[:, None], s, -1)
        assert np.all(pad == -1)


def full_check(q, k, v, B, topk, rows=None, gpu=None):
    """GPU forward vs oracle on all rows (or the given (rows_t, rows_h))."""
    S, Hq, _ = q.shape
    Hkv = k.shape[1]
    out_g, lse_g, sel_g, kmean_g = run_gpu(q, k, v, B, topk) if gpu is None else gpu
    nbp = oracle.nblocks(S, B) - 1
    k_eff = min(topk, nbp + 1)
    m = oracle.kmean(k, B)
    if nbp > 0 and 1 < k_eff < nbp + 1:
        np.testing.assert_allclose(kmean_g, m[:, :nbp], rtol=1e-5, atol=1e-5)
    check_sel_structure(sel_g, S, B, topk)
    if rows is None:
        rows_t, rows_h = oracle.all_rows(S, Hq)
    else:
        rows_t, rows_h = rows
    sel_rows = sel_g[rows_h, rows_t]
    sel_acc, n_near = check_selection(q, k, sel_rows, rows_t, rows_h, B, Hkv, topk, m)
    out_o, lse_o, _ = oracle.attend(q, k, v, B, topk, rows_t, rows_h, sel=sel_acc)
    out_rows = out_g[torch.from_numpy(rows_t), torch.from_numpy(rows_h.astype(np.int64))].float().numpy()
    stats = compare_outputs(out_rows, lse_g[rows_h, rows_t], out_o, lse_o)
    stats["near_ties"] = n_near
    return stats
