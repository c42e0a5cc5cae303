"""Seeded synthetic inputs for the MoBA causal prefill forward pass.

This module only draws random numbers (counter-based SplitMix64 + Box-Muller,
rounded to bf16) and defines the workloads. It holds none of the attention
method's arithmetic, so both the fp64 oracle and the CUDA path can take their
inputs from it without sharing any of the method's code.

Workloads (batch 1, head_dim 128): Q, K, V are i.i.d. N(0, 1) in bf16, and
every key of block j of kv head g also carries the offset mu[g][j] of norm
0.5*sqrt(128), so gate scores separate (the mixture-of-block-attention
abstract, arXiv 2502.13189: a parameter-less top-k gate per query picks the
most relevant KV blocks).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libsynth.so")

STREAM_Q, STREAM_K, STREAM_V, STREAM_MU, STREAM_DO = 1, 2, 3, 4, 5


@dataclass(frozen=True)
class Workload:
    name: str
    seqlen: int
    heads_q: int
    heads_kv: int
    head_dim: int
    block_size: int
    topk: int
    seed: int

    @property
    def nblocks(self) -> int:
        return (self.seqlen + self.block_size - 1) // self.block_size


# Five workloads, seed 20250218 + index. The 32K one is the shape of the
# micro-benchmark on the MoBA project page (32K tokens, 1 head, block 2048,
# top-3); the 128K/1M ones use the Llama-3.1-8B attention shape (32 q heads,
# 8 kv heads); the 10M one is the longest context the pages mention.
WORKLOADS = {
    "4k": Workload("moba_4k_h1_b512_k3", 4096, 1, 1, 128, 512, 3, 20250218 + 0),
    "32k": Workload("moba_32k_h1_b2048_k3", 32768, 1, 1, 128, 2048, 3, 20250218 + 1),
    "128k": Workload("moba_128k_h32kv8_b4096_k12", 131072, 32, 8, 128, 4096, 12, 20250218 + 2),
    "1m": Workload("moba_1m_h32kv8_b4096_k12", 1048576, 32, 8, 128, 4096, 12, 20250218 + 3),
    "10m": Workload("moba_10m_h1_b8192_k12", 10485760, 1, 1, 128, 8192, 12, 20250218 + 4),
    # topk >= number of blocks: full causal attention (the dense path), on the
    # inputs of the 32K and 128K workloads
    "32k_dense": Workload("moba_32k_h1_b2048_k16_dense", 32768, 1, 1, 128, 2048, 16, 20250218 + 1),
    "128k_dense": Workload("moba_128k_h32kv8_b4096_k32_dense", 131072, 32, 8, 128, 4096, 32, 20250218 + 2),
    # finer blocks: 512-token blocks, top-48 (about the 128K workload's
    # selected keys per query), on the 128K workload's seed
    "128k_b512": Workload("moba_128k_h32kv8_b512_k48", 131072, 32, 8, 128, 512, 48, 20250218 + 2),
}


def _build() -> None:
    if os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-pthread", "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB)


_lib = None


def lib():
    global _lib
    if _lib is None:
        _build()
        L = ctypes.CDLL(_LIB)
        u64, i64, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p
        L.synth_stream_state.restype = u64
        L.synth_stream_state.argtypes = [u64, u64]
        L.synth_splitmix_output.restype = u64
        L.synth_splitmix_output.argtypes = [u64, u64]
        L.synth_normal.restype = ctypes.c_double
        L.synth_normal.argtypes = [u64, u64, u64]
        L.synth_f64_to_bf16.restype = ctypes.c_uint16
        L.synth_f64_to_bf16.argtypes = [ctypes.c_double]
        L.synth_fill_normal_bf16.restype = None
        L.synth_fill_normal_bf16.argtypes = [vp, i64, u64, u64, i64, ctypes.c_int]
        L.synth_key_offsets.restype = None
        L.synth_key_offsets.argtypes = [vp, i64, i64, i64, u64, u64]
        L.synth_fill_keys_bf16.restype = None
        L.synth_fill_keys_bf16.argtypes = [vp, i64, i64, i64, i64, i64, i64, vp, u64, u64, ctypes.c_int]
        _lib = L
    return _lib


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def key_offsets(w: Workload) -> np.ndarray:
    mu = np.empty((w.heads_kv, w.nblocks, w.head_dim), dtype=np.float64)
    lib().synth_key_offsets(mu.ctypes.data, w.heads_kv, w.nblocks, w.head_dim, w.seed, STREAM_MU)
    return mu


def fill_q(ptr: int, w: Workload, t0: int = 0, nrows: int | None = None, threads: int | None = None) -> None:
    """Write bf16 Q rows [t0, t0+nrows) of a [S][Hq][d] tensor to host memory at ptr."""
    nrows = w.seqlen - t0 if nrows is None else nrows
    per = w.heads_q * w.head_dim
    lib().synth_fill_normal_bf16(ptr, nrows * per, w.seed, STREAM_Q, t0 * per, threads or default_threads())


def fill_v(ptr: int, w: Workload, t0: int = 0, nrows: int | None = None, threads: int | None = None) -> None:
    nrows = w.seqlen - t0 if nrows is None else nrows
    per = w.heads_kv * w.head_dim
    lib().synth_fill_normal_bf16(ptr, nrows * per, w.seed, STREAM_V, t0 * per, threads or default_threads())


def fill_dout(ptr: int, w: Workload, t0: int = 0, nrows: int | None = None, threads: int | None = None) -> None:
    """Upstream gradient dO [S][Hq][d] for the backward pass: i.i.d. N(0, 1) bf16."""
    nrows = w.seqlen - t0 if nrows is None else nrows
    per = w.heads_q * w.head_dim
    lib().synth_fill_normal_bf16(ptr, nrows * per, w.seed, STREAM_DO, t0 * per, threads or default_threads())


def make_dout(w: Workload, threads: int | None = None) -> np.ndarray:
    """Host numpy uint16 (bf16 bit patterns) dO [S,Hq,d]."""
    do = np.empty((w.seqlen, w.heads_q, w.head_dim), dtype=np.uint16)
    fill_dout(do.ctypes.data, w, threads=threads)
    return do


def fill_k(ptr: int, w: Workload, mu: np.ndarray | None = None, t0: int = 0, nrows: int | None = None,
           threads: int | None = None) -> None:
    nrows = w.seqlen - t0 if nrows is None else nrows
    mu = key_offsets(w) if mu is None else np.ascontiguousarray(mu, dtype=np.float64)
    lib().synth_fill_keys_bf16(ptr, t0, nrows, w.heads_kv, w.head_dim, w.block_size, w.nblocks,
                               mu.ctypes.data, w.seed, STREAM_K, threads or default_threads())


def make_qkv(w: Workload, threads: int | None = None):
    """Host numpy uint16 (bf16 bit patterns) arrays q [S,Hq,d], k, v [S,Hkv,d]."""
    q = np.empty((w.seqlen, w.heads_q, w.head_dim), dtype=np.uint16)
    k = np.empty((w.seqlen, w.heads_kv, w.head_dim), dtype=np.uint16)
    v = np.empty((w.seqlen, w.heads_kv, w.head_dim), dtype=np.uint16)
    fill_q(q.ctypes.data, w, threads=threads)
    fill_k(k.ctypes.data, w, threads=threads)
    fill_v(v.ctypes.data, w, threads=threads)
    return q, k, v


def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even of float64 values to bf16 bit patterns (uint16)."""
    L = lib()
    flat = np.asarray(x, dtype=np.float64).ravel()
    out = np.fromiter((L.synth_f64_to_bf16(float(v)) for v in flat), dtype=np.uint16, count=flat.size)
    return out.reshape(np.shape(x))
