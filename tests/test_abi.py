"""The C-ABI library: it builds, loads, exports every entry point that
include/moba.h declares, and rejects bad arguments before touching a GPU."""
import ctypes
import os
import re

import pytest

import block_sparse_long_fwd_b200 as moba
from block_sparse_long_fwd_b200 import build as moba_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_entry_points():
    src = open(os.path.join(ROOT, "include", "moba.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(moba_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    moba_build.build()
    return moba.lib()


def test_header_declares_the_expected_calls():
    names = declared_entry_points()
    assert "moba_fwd" in names and "moba_last_error" in names
    assert set(names) == set(moba.SIGNATURES), names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_entry_points():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


FAKE = 0x1000  # 16-byte aligned, never dereferenced: checks fail first


@pytest.mark.parametrize("args,code", [
    # q, k, v, S, Hq, Hkv, d, B, topk, out, lse
    ((0, FAKE, FAKE, 4096, 1, 1, 128, 512, 3, FAKE, FAKE), moba.MOBA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, 0, 1, 1, 128, 512, 3, FAKE, FAKE), moba.MOBA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, 4096, 3, 2, 128, 512, 3, FAKE, FAKE), moba.MOBA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, 4096, 1, 1, 64, 512, 3, FAKE, FAKE), moba.MOBA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, 4096, 1, 1, 128, 500, 3, FAKE, FAKE), moba.MOBA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, 4096, 1, 1, 128, 0, 3, FAKE, FAKE), moba.MOBA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, 4096, 1, 1, 128, 512, 0, FAKE, FAKE), moba.MOBA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, 4096, 0, 1, 128, 512, 3, FAKE, FAKE), moba.MOBA_ERR_INVALID_ARG),
    ((FAKE + 8, FAKE, FAKE, 4096, 1, 1, 128, 512, 3, FAKE, FAKE), moba.MOBA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, 1 << 20, 1, 1, 128, 128, 100, FAKE, FAKE), moba.MOBA_ERR_UNSUPPORTED),
    ((FAKE, FAKE, FAKE, 1 << 20, 1, 1, 128, 128, 66, FAKE, FAKE), moba.MOBA_ERR_UNSUPPORTED),  # 65 past blocks
])
def test_invalid_arguments_are_rejected_before_launch(lib, args, code):
    rc = lib.moba_fwd(*args, None)
    assert rc == code
    assert moba.last_error()


def test_error_message_is_thread_local_and_cleared(lib):
    assert lib.moba_fwd(0, 0, 0, 1, 1, 1, 128, 128, 1, 0, 0, None) == moba.MOBA_ERR_INVALID_ARG
    assert "null" in moba.last_error()


def test_without_a_gpu_valid_calls_fail_loudly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    rc = lib.moba_fwd(FAKE, FAKE, FAKE, 4096, 1, 1, 128, 512, 3, FAKE, FAKE, None)
    assert rc == moba.MOBA_ERR_CUDA
    with pytest.raises(ValueError):
        moba.fwd(torch.zeros(4, 1, 128, dtype=torch.bfloat16), torch.zeros(4, 1, 128, dtype=torch.bfloat16),
                 torch.zeros(4, 1, 128, dtype=torch.bfloat16), 128, 1)


def test_effective_flops_counts_selected_pairs():
    # S = 3 blocks of 2 tokens (B = 2), topk 2: own block causal + 1 past block
    # (mirrors the per-query key count min(k-1, b) * B + (t mod B) + 1)
    S, B, k = 6, 2, 2
    pairs = sum(min(k - 1, t // B) * B + t % B + 1 for t in range(S))
    assert moba.effective_flops(S, 1, B, k, head_dim=1) == 4 * pairs


@pytest.mark.parametrize("q_start", [-1, 4096, 5000])
def test_chunk_rejects_a_query_start_outside_the_sequence(lib, q_start):
    rc = lib.moba_fwd_chunk(FAKE, FAKE, FAKE, 4096, q_start, 1, 1, 128, 512, 3, FAKE, FAKE, None)
    assert rc == moba.MOBA_ERR_INVALID_ARG
    assert "q_start" in moba.last_error()


def test_chunk_with_means_rejects_null_means(lib):
    rc = lib.moba_fwd_chunk_means(FAKE, FAKE, FAKE, None, 4096, 4000, 1, 1, 128, 512, 3, FAKE, FAKE, None)
    assert rc == moba.MOBA_ERR_INVALID_ARG
    assert "kmean" in moba.last_error()


def _cu(vals):
    arr = (ctypes.c_int64 * len(vals))(*vals)
    return arr, len(vals) - 1


@pytest.mark.parametrize("cu, what", [
    ([1, 4096], "cu_seqlens[0]"),
    ([0, 4096, 2048], "non-decreasing"),
    ([0, 0, 0], "no tokens"),
    ([0], "batch"),
])
def test_varlen_rejects_bad_offsets_before_launch(lib, cu, what):
    arr, batch = _cu(cu)
    rc = lib.moba_fwd_varlen(FAKE, FAKE, FAKE, ctypes.cast(arr, ctypes.c_void_p), batch, 1, 1, 128, 512, 3, FAKE,
                             FAKE, None)
    assert rc == moba.MOBA_ERR_INVALID_ARG
    assert what in moba.last_error()


def test_varlen_checks_each_sequence_shape_and_pointers(lib):
    arr, batch = _cu([0, 4096, 8192])
    rc = lib.moba_fwd_varlen(FAKE, FAKE, FAKE, None, batch, 1, 1, 128, 512, 3, FAKE, FAKE, None)
    assert rc == moba.MOBA_ERR_INVALID_ARG and "null" in moba.last_error()
    # lse only needs 4-byte alignment (a sequence's lse columns start anywhere)
    rc = lib.moba_fwd_varlen(FAKE, FAKE, FAKE, ctypes.cast(arr, ctypes.c_void_p), batch, 1, 1, 128, 512, 3, FAKE,
                             FAKE + 2, None)
    assert rc == moba.MOBA_ERR_INVALID_ARG and "lse" in moba.last_error()
    rc = lib.moba_fwd_varlen(FAKE, FAKE, FAKE, ctypes.cast(arr, ctypes.c_void_p), batch, 3, 2, 128, 512, 3, FAKE,
                             FAKE + 4, None)
    assert rc == moba.MOBA_ERR_INVALID_ARG and "multiple" in moba.last_error()


def test_backward_rejects_bad_arguments_before_launch(lib):
    rc = lib.moba_bwd(FAKE, FAKE, FAKE, FAKE, None, FAKE, 4096, 1, 1, 128, 512, 3, FAKE, FAKE, FAKE, None)
    assert rc == moba.MOBA_ERR_INVALID_ARG and "null" in moba.last_error()
    rc = lib.moba_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4096, 1, 1, 64, 512, 3, FAKE, FAKE, FAKE, None)
    assert rc == moba.MOBA_ERR_INVALID_ARG and "head_dim" in moba.last_error()
    rc = lib.moba_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 8, 4096, 1, 1, 128, 512, 3, FAKE, FAKE, FAKE, None)
    assert rc == moba.MOBA_ERR_INVALID_ARG and "aligned" in moba.last_error()


def test_async_selftest_checks_its_bound_before_launch(lib):
    assert lib.moba_selftest_bounded_wait_async(0, None) == moba.MOBA_ERR_INVALID_ARG
    assert lib.moba_selftest_bounded_wait_async(3000000, None) == moba.MOBA_ERR_INVALID_ARG
