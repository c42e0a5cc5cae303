"""B200 (sm_100a) MoBA causal prefill forward pass: thin Python binding.

Every step of the forward pass (key mean-pool, gate + top-k, router, block
attention, log-sum-exp merge) runs in the CUDA kernels of the C-ABI library
``libmoba_b200.so`` declared in ``include/moba.h``. This module only passes
pointers, sizes and the current torch stream to it; PyTorch supplies device
memory and streams. There is no CPU fallback: when the library is missing the
calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoba_b200.so")

MOBA_OK = 0
MOBA_ERR_INVALID_ARG = 1
MOBA_ERR_UNSUPPORTED = 2
MOBA_ERR_OOM = 3
MOBA_ERR_CUDA = 4
MOBA_ERR_DEVICE_TIMEOUT = 5
MOBA_ERR_DEVICE_CHECK = 6
HEAD_DIM = 128
MAX_TOPK = 64

# every entry point the header declares, with its ctypes signature
_vp, _i64, _i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
SIGNATURES = {
    "moba_fwd": (_i32, [_vp, _vp, _vp, _i64, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moba_fwd_chunk": (_i32, [_vp, _vp, _vp, _i64, _i64, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moba_fwd_chunk_means": (_i32, [_vp, _vp, _vp, _vp, _i64, _i64, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moba_fwd_varlen": (_i32, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moba_bwd": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp]),
    "moba_fwd_host": (_i32, [_vp, _vp, _vp, _i64, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moba_pool": (_i32, [_vp, _i64, _i32, _i32, _i32, _vp, _vp]),
    "moba_gate": (_i32, [_vp, _vp, _i64, _i32, _i32, _i32, _i32, _i32, _vp, _vp]),
    "moba_fwd_noalloc": (_i32, [_vp, _vp, _vp, _i64, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moba_profile_begin": (_i32, []),
    "moba_profile_end": (_i32, [_vp, _vp, _vp]),
    "moba_last_error": (ctypes.c_char_p, []),
    "moba_device_status": (_i32, [_vp]),
    "moba_selftest_bounded_wait": (_i32, [_i32, _vp]),
    "moba_selftest_bounded_wait_async": (_i32, [_i32, _vp]),
    "moba_selftest_device_check": (_i32, [_vp]),
}


class MobaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"moba status {code}: {msg}")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C-ABI library. Raises when it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m block_sparse_long_fwd_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def last_error() -> str:
    return lib().moba_last_error().decode()


def _check(rc: int) -> None:
    if rc != MOBA_OK:
        raise MobaError(rc, last_error())


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _dev_bf16(x: torch.Tensor, name: str) -> torch.Tensor:
    if not (x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    return x


def nblocks(seqlen: int, block_size: int) -> int:
    return (seqlen + block_size - 1) // block_size


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block_size: int, topk: int, out=None, lse=None,
        stream=None):
    """MoBA forward. q [S,Hq,128], k/v [S,Hkv,128] bf16 on the GPU.

    Returns (out [S,Hq,128] bf16, lse [Hq,S] fp32), queued on ``stream``
    (default: the current torch stream).
    """
    _dev_bf16(q, "q"), _dev_bf16(k, "k"), _dev_bf16(v, "v")
    S, Hq, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (S, Hkv, d) or v.shape != k.shape:
        raise ValueError("k and v must be [S, heads_kv, head_dim] matching q")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((Hq, S), dtype=torch.float32, device=q.device)
    _check(lib().moba_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), S, Hq, Hkv, d, block_size, topk,
                          out.data_ptr(), lse.data_ptr(), _stream(stream)))
    return out, lse


def fwd_chunk(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block_size: int, topk: int, out=None, lse=None,
              stream=None, kmean=None):
    """MoBA forward for the last n = q.shape[0] tokens of a sequence of
    S = k.shape[0] tokens (chunked prefill; n = 1 is a decode step).

    q [n,Hq,128] holds the queries of tokens S-n .. S-1; k/v [S,Hkv,128] the
    keys and values of all S tokens. Returns (out [n,Hq,128] bf16,
    lse [Hq,n] fp32), equal to those rows of ``fwd`` on the whole sequence.
    """
    _dev_bf16(q, "q"), _dev_bf16(k, "k"), _dev_bf16(v, "v")
    n, Hq, d = q.shape
    S, Hkv = k.shape[0], k.shape[1]
    if v.shape != k.shape or k.shape[2] != d or not 1 <= n <= S:
        raise ValueError("q must be [n, heads_q, head_dim] with 1 <= n <= S; k and v [S, heads_kv, head_dim]")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((Hq, n), dtype=torch.float32, device=q.device)
    if kmean is not None:
        # block means from pool() for these k and block_size, kept by the caller
        if kmean.dtype != torch.float32 or not kmean.is_cuda or not kmean.is_contiguous():
            raise ValueError("kmean must be a contiguous fp32 CUDA tensor from pool()")
        _check(lib().moba_fwd_chunk_means(q.data_ptr(), k.data_ptr(), v.data_ptr(), kmean.data_ptr(), S, S - n, Hq,
                                          Hkv, d, block_size, topk, out.data_ptr(), lse.data_ptr(), _stream(stream)))
        return out, lse
    _check(lib().moba_fwd_chunk(q.data_ptr(), k.data_ptr(), v.data_ptr(), S, S - n, Hq, Hkv, d, block_size, topk,
                                out.data_ptr(), lse.data_ptr(), _stream(stream)))
    return out, lse


def fwd_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens, block_size: int, topk: int, out=None,
               lse=None, stream=None):
    """MoBA forward over a packed batch of independent sequences.

    q [T,Hq,128], k/v [T,Hkv,128] bf16 on the GPU hold the sequences one after
    another; ``cu_seqlens`` (a sequence of ints or a CPU tensor, length
    batch + 1, starting at 0) gives their offsets. Returns (out [T,Hq,128]
    bf16, lse [Hq,T] fp32); sequence b's rows equal ``fwd`` on its tokens.
    """
    _dev_bf16(q, "q"), _dev_bf16(k, "k"), _dev_bf16(v, "v")
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (T, Hkv, d) or v.shape != k.shape:
        raise ValueError("k and v must be [T, heads_kv, head_dim] matching q")
    cu = torch.as_tensor(cu_seqlens, dtype=torch.int64, device="cpu").contiguous()
    if cu.dim() != 1 or cu.numel() < 2 or int(cu[-1]) != T:
        raise ValueError("cu_seqlens must be 1-D with batch + 1 entries ending at q.shape[0]")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((Hq, T), dtype=torch.float32, device=q.device)
    _check(lib().moba_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), cu.data_ptr(), cu.numel() - 1, Hq, Hkv, d,
                                 block_size, topk, out.data_ptr(), lse.data_ptr(), _stream(stream)))
    return out, lse


def bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor, lse: torch.Tensor,
        dout: torch.Tensor, block_size: int, topk: int, stream=None):
    """Gradient of ``fwd`` with the gate's choice held fixed.

    q [S,Hq,128], k/v [S,Hkv,128], out and dout [S,Hq,128] bf16 and lse
    [Hq,S] fp32 (``fwd``'s outputs) on the GPU. Returns (dq, dk, dv) bf16.
    """
    for name, x in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout)):
        _dev_bf16(x, name)
    S, Hq, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (S, Hkv, d) or v.shape != k.shape or out.shape != q.shape or dout.shape != q.shape:
        raise ValueError("k, v must be [S, heads_kv, head_dim]; out and dout [S, heads_q, head_dim]")
    if lse.dtype != torch.float32 or not lse.is_cuda or not lse.is_contiguous() or lse.shape != (Hq, S):
        raise ValueError("lse must be a contiguous fp32 CUDA tensor [heads_q, S]")
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    _check(lib().moba_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), dout.data_ptr(),
                          S, Hq, Hkv, d, block_size, topk, dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                          _stream(stream)))
    return dq, dk, dv


STAGES = ("pool", "gate", "route", "attention", "merge", "bwd_prep", "bwd_dq", "bwd_dkdv")


def profile_begin() -> None:
    """Start per-stage device timing of the forward calls from this thread."""
    _check(lib().moba_profile_begin())


def profile_end():
    """Stop timing; returns ({stage: total ms}, kernel launches, forward calls)."""
    ms = (ctypes.c_float * len(STAGES))()
    n, c = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().moba_profile_end(ms, ctypes.byref(n), ctypes.byref(c)))
    return dict(zip(STAGES, list(ms))), n.value, c.value


def fwd_host(q, k, v, block_size: int, topk: int, out=None, lse=None, stream=None):
    """MoBA forward on HOST tensors (bf16 torch CPU tensors, pinned for speed).

    The library copies inputs to the device, runs the pass, copies out/lse
    back and synchronises the stream.
    """
    S, Hq, d = q.shape
    Hkv = k.shape[1]
    for name, x in (("q", q), ("k", k), ("v", v)):
        if x.is_cuda or x.dtype != torch.bfloat16 or not x.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CPU tensor")
    if out is None:
        out = torch.empty((S, Hq, d), dtype=torch.bfloat16, pin_memory=q.is_pinned())
    if lse is None:
        lse = torch.empty((Hq, S), dtype=torch.float32, pin_memory=q.is_pinned())
    _check(lib().moba_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), S, Hq, Hkv, d, block_size, topk,
                               out.data_ptr(), lse.data_ptr(), _stream(stream)))
    return out, lse


def pool(k: torch.Tensor, block_size: int, stream=None) -> torch.Tensor:
    """Key mean-pool stage alone: fp32 [Hkv, nblocks-1, 128]."""
    _dev_bf16(k, "k")
    S, Hkv, d = k.shape
    nbp = max(nblocks(S, block_size) - 1, 0)
    kmean = torch.empty((Hkv, max(nbp, 1), d), dtype=torch.float32, device=k.device)
    _check(lib().moba_pool(k.data_ptr(), S, Hkv, d, block_size, kmean.data_ptr(), _stream(stream)))
    return kmean[:, :nbp]


def gate(q: torch.Tensor, kmean: torch.Tensor, heads_kv: int, block_size: int, topk: int, stream=None):
    """Gate + top-k stage alone: int32 sel [Hq, S, min(topk, nblocks)]."""
    _dev_bf16(q, "q")
    S, Hq, d = q.shape
    k_eff = min(topk, nblocks(S, block_size))
    sel = torch.empty((Hq, S, k_eff), dtype=torch.int32, device=q.device)
    kp = kmean.data_ptr() if kmean is not None and kmean.numel() else None
    _check(lib().moba_gate(q.data_ptr(), kp, S, Hq, heads_kv, d, block_size, topk, sel.data_ptr(),
                           _stream(stream)))
    return sel


def device_status(stream=None) -> int:
    """Synchronise the stream, return and clear the kernels' status word."""
    return lib().moba_device_status(_stream(stream))


def selftest_bounded_wait(timeout_us: int = 20000, stream=None) -> int:
    return lib().moba_selftest_bounded_wait(timeout_us, _stream(stream))


def effective_flops(seqlen: int, heads_q: int, block_size: int, topk: int, head_dim: int = HEAD_DIM) -> float:
    """Selected-block FLOPs: 4*d*Hq per unmasked (query, key) pair.

    A query t attends min(topk-1, t//B) full past blocks plus the keys of its
    own block up to itself.
    """
    nb = nblocks(seqlen, block_size)
    k_eff = min(topk, nb)
    pairs = 0
    for b in range(nb):
        t0, t1 = b * block_size, min(seqlen, (b + 1) * block_size)
        n = t1 - t0
        pairs += n * min(k_eff - 1, b) * block_size + n * (n + 1) // 2
    return 4.0 * head_dim * heads_q * pairs
