"""fp64 CPU oracle for the MoBA causal prefill forward pass.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use it. The product path (the CUDA library and
its binding) never imports it, and it imports nothing from the product path.

The arithmetic lives in ``moba_oracle.c`` (plain loops, fp64, threads over
rows). This wrapper only compiles it with gcc and marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moba_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")


def build() -> str:
    if os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    # -O3 without -ffast-math: IEEE double arithmetic in the order written
    subprocess.check_call(["gcc", "-O3", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared", "-pthread", "-o",
                           tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.oracle_kmean.restype = None
        L.oracle_kmean.argtypes = [vp, i64, i32, i32, i32, vp]
        L.oracle_gate_scores.restype = None
        L.oracle_gate_scores.argtypes = [vp, vp, i64, i32, i32, i32, i32, i64, i32, vp]
        L.oracle_select.restype = None
        L.oracle_select.argtypes = [vp, vp, i64, i32, i32, i32, i32, i32, vp, vp, i64, vp, vp, i32]
        L.oracle_attend.restype = None
        L.oracle_attend.argtypes = [vp, vp, vp, vp, i64, i32, i32, i32, i32, i32, vp, vp, i64, vp, vp, vp,
                                    vp, i32]
        _lib = L
    return _lib


def threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _u16(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("expected bf16 bit patterns as uint16")
    return a


def nblocks(S: int, B: int) -> int:
    return (S + B - 1) // B


def kmean(k: np.ndarray, block_size: int) -> np.ndarray:
    """Mean-pooled keys, fp64 [Hkv][nb][d]. k: uint16 [S][Hkv][d]."""
    k = _u16(k)
    S, Hkv, d = k.shape
    m = np.empty((Hkv, nblocks(S, block_size), d), dtype=np.float64)
    lib().oracle_kmean(k.ctypes.data, S, Hkv, d, block_size, m.ctypes.data)
    return m


def gate_scores(q: np.ndarray, m: np.ndarray, block_size: int, heads_kv: int, t: int, h: int) -> np.ndarray:
    """Scores of row (t, h) against its past blocks j < t // block_size."""
    q = _u16(q)
    S, Hq, d = q.shape
    m = np.ascontiguousarray(m, dtype=np.float64)
    s = np.empty(max(1, t // block_size), dtype=np.float64)
    lib().oracle_gate_scores(q.ctypes.data, m.ctypes.data, S, Hq, heads_kv, d, block_size, t, h, s.ctypes.data)
    return s[: t // block_size]


def _rows(rows_t, rows_h):
    rt = np.ascontiguousarray(rows_t, dtype=np.int64)
    rh = np.ascontiguousarray(rows_h, dtype=np.int32)
    if rt.shape != rh.shape or rt.ndim != 1:
        raise ValueError("rows_t and rows_h must be 1-D and of equal length")
    return rt, rh


def all_rows(S: int, Hq: int):
    """(t, h) for every row, t-major."""
    t = np.repeat(np.arange(S, dtype=np.int64), Hq)
    h = np.tile(np.arange(Hq, dtype=np.int32), S)
    return t, h


def select(q: np.ndarray, m: np.ndarray, block_size: int, heads_kv: int, topk: int, rows_t, rows_h,
           nthreads: int | None = None):
    """Selected blocks per row: (sel int32 [n][k_eff] ascending, -1 padded; info fp64 [n][4]).

    info[:, 0] is the gap at the cut relative to the row's largest |score|,
    info[:, 1] the last chosen past score, info[:, 2] the first left out,
    info[:, 3] the row's largest |score| over its past blocks."""
    q = _u16(q)
    S, Hq, d = q.shape
    m = np.ascontiguousarray(m, dtype=np.float64)
    rt, rh = _rows(rows_t, rows_h)
    k_eff = min(topk, nblocks(S, block_size))
    sel = np.empty((rt.size, k_eff), dtype=np.int32)
    info = np.empty((rt.size, 4), dtype=np.float64)
    lib().oracle_select(q.ctypes.data, m.ctypes.data, S, Hq, heads_kv, d, block_size, topk, rt.ctypes.data,
                        rh.ctypes.data, rt.size, sel.ctypes.data, info.ctypes.data, nthreads or threads())
    return sel, info


def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, block_size: int, topk: int, rows_t=None, rows_h=None,
           sel: np.ndarray | None = None, m: np.ndarray | None = None, nthreads: int | None = None):
    """MoBA forward for the given rows (all rows when omitted).

    Returns (out fp64 [n][d], lse fp64 [n], sel int32 [n][k_eff]). When ``sel``
    is given, it replaces the gate for those rows.
    """
    q, k, v = _u16(q), _u16(k), _u16(v)
    S, Hq, d = q.shape
    Hkv = k.shape[1]
    if rows_t is None:
        rows_t, rows_h = all_rows(S, Hq)
    rt, rh = _rows(rows_t, rows_h)
    k_eff = min(topk, nblocks(S, block_size))
    out = np.empty((rt.size, d), dtype=np.float64)
    lse = np.empty(rt.size, dtype=np.float64)
    sel_out = np.empty((rt.size, k_eff), dtype=np.int32)
    if sel is not None:
        sel_in = np.ascontiguousarray(sel, dtype=np.int32)
        if sel_in.shape != (rt.size, k_eff):
            raise ValueError(f"sel must be [{rt.size}][{k_eff}]")
        sel_out[...] = sel_in
        mp = None
        sp = sel_in.ctypes.data
    else:
        m = kmean(k, block_size) if m is None else np.ascontiguousarray(m, dtype=np.float64)
        mp = m.ctypes.data
        sp = None
    lib().oracle_attend(q.ctypes.data, k.ctypes.data, v.ctypes.data, mp, S, Hq, Hkv, d, block_size, topk,
                        rt.ctypes.data, rh.ctypes.data, rt.size, sp, None if sel is not None else sel_out.ctypes.data,
                        out.ctypes.data, lse.ctypes.data, nthreads or threads())
    return out, lse, sel_out
