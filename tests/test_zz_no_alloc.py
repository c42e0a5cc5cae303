"""moba_fwd_noalloc: the forward pass without any device allocation.

Some callers may not allocate device memory while they run: a serving process
that reserved its whole memory budget at start-up, or a plug-in that sits
under an allocator it does not own. moba_fwd_noalloc serves them from one
fixed device array inside the library. These tests call it through the C ABI
and check it against moba_fwd, the stream-ordered entry point, with the
tolerances the other parity tests use, on two calls in a row (the second
call finds the array holding the first call's contents).

The file name sorts last so that a run that stops at the first failure has
already run every other test.
"""
import numpy as np
import pytest

import oracle
from parity_helpers import (LSE_ABS, OUT_MAX_ABS, OUT_MEAN_ABS, check_selection, compare_outputs, make_inputs,
                            to_dev)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

import block_sparse_long_fwd_b200 as moba  # noqa: E402


def call(fn_name, q, k, v, B, topk):
    S, Hq, d = q.shape
    Hkv = k.shape[1]
    out = torch.empty_like(q)
    lse = torch.empty((Hq, S), dtype=torch.float32, device=q.device)
    fn = getattr(moba.lib(), fn_name)
    rc = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), S, Hq, Hkv, d, B, topk, out.data_ptr(), lse.data_ptr(),
            torch.cuda.current_stream().cuda_stream)
    assert rc == moba.MOBA_OK, (fn_name, rc, moba.last_error())
    return out, lse


def close(a, b):
    (oa, la), (ob, lb) = a, b
    err = (oa.float() - ob.float()).abs()
    assert err.max().item() <= OUT_MAX_ABS and err.mean().item() <= OUT_MEAN_ABS
    assert (la - lb).abs().max().item() <= LSE_ABS


@pytest.mark.parametrize("S,Hq,Hkv,B,topk,seed", [
    (4096, 1, 1, 512, 3, 1),     # the small workload's shape
    (3000, 4, 2, 256, 5, 2),     # GQA, ragged tail, several routed blocks
    (32768, 1, 1, 2048, 3, 3),   # the project page's micro-benchmark shape
])
def test_matches_stream_ordered_entry_point_twice(S, Hq, Hkv, B, topk, seed):
    _, q, k, v = make_inputs(S, Hq, Hkv, B, topk, seed)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    ref = call("moba_fwd", qd, kd, vd, B, topk)
    first = call("moba_fwd_noalloc", qd, kd, vd, B, topk)
    second = call("moba_fwd_noalloc", qd, kd, vd, B, topk)
    torch.cuda.synchronize()
    assert moba.device_status() == moba.MOBA_OK
    close(first, ref)
    close(second, ref)


def test_other_inputs_after_a_previous_call():
    # the array keeps the previous call's contents; a new problem must not see them
    _, q1, k1, v1 = make_inputs(2048, 2, 1, 256, 4, 11)
    _, q2, k2, v2 = make_inputs(1536, 4, 4, 128, 3, 12)
    call("moba_fwd_noalloc", to_dev(q1), to_dev(k1), to_dev(v1), 256, 4)
    q2d, k2d, v2d = to_dev(q2), to_dev(k2), to_dev(v2)
    got = call("moba_fwd_noalloc", q2d, k2d, v2d, 128, 3)
    ref = call("moba_fwd", q2d, k2d, v2d, 128, 3)
    torch.cuda.synchronize()
    assert moba.device_status() == moba.MOBA_OK
    close(got, ref)


def test_a_problem_that_needs_several_query_windows():
    # The selection table (32768 x 16 x 8 x 4 B = 16.8 MB) fits in the fixed
    # array but a whole-sequence query window (~0.9 GB of partial outputs)
    # does not: the call must shrink its window and run several of them.
    S, Hq, Hkv, B, topk = 32768, 16, 4, 2048, 8
    _, q, k, v = make_inputs(S, Hq, Hkv, B, topk, 21)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    moba.profile_begin()
    got = call("moba_fwd_noalloc", qd, kd, vd, B, topk)
    _, launches, calls = moba.profile_end()
    # pool and gate (3 kernels), then per window the router (1 kernel while the
    # window holds no past block, else 4), attention and merge: one window
    # would be at most 9 launches (1024-token windows here: 189)
    assert calls == 1 and launches > 9, launches
    again = call("moba_fwd_noalloc", qd, kd, vd, B, topk)
    ref = call("moba_fwd", qd, kd, vd, B, topk)
    torch.cuda.synchronize()
    assert moba.device_status() == moba.MOBA_OK
    close(got, ref)
    close(again, ref)
    # and against the oracle on drawn rows of every head
    rng = np.random.default_rng(5)
    rows_t = rng.choice(S, size=512, replace=False).astype(np.int64)
    rows_h = (np.arange(512) % Hq).astype(np.int32)
    sel = moba.gate(qd, moba.pool(kd, B), Hkv, B, topk).cpu().numpy()[rows_h, rows_t]
    sel, _ = check_selection(q, k, sel, rows_t, rows_h, B, Hkv, topk)
    out_o, lse_o, _ = oracle.attend(q, k, v, B, topk, rows_t, rows_h, sel=sel)
    out, lse = got
    compare_outputs(out[torch.from_numpy(rows_t), torch.from_numpy(rows_h.astype(np.int64))].float().cpu().numpy(),
                    lse.cpu().numpy()[rows_h, rows_t], out_o, lse_o)


def test_rejects_problems_beyond_the_fixed_scratch():
    # 262144 tokens x 8 heads x top-8: the selection table alone (67 MB)
    # exceeds the fixed array. Real, correctly sized buffers: were the check
    # ever to let the call through, it would compute a valid result instead of
    # touching memory it does not own, and fail the assertion below.
    S, Hq, Hkv, B, topk = 262144, 8, 1, 128, 8
    q = torch.zeros((S, Hq, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((S, Hkv, 128), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    out = torch.empty_like(q)
    lse = torch.empty((Hq, S), dtype=torch.float32, device="cuda")
    rc = moba.lib().moba_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), S, Hq, Hkv, 128, B, topk,
                                     out.data_ptr(), lse.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == moba.MOBA_ERR_UNSUPPORTED
    assert "too large for moba_fwd_noalloc" in moba.last_error()
    torch.cuda.synchronize()
    assert moba.device_status() == moba.MOBA_OK
