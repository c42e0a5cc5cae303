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
import ctypes

import numpy as np
import pytest

from parity_helpers import LSE_ABS, OUT_MAX_ABS, OUT_MEAN_ABS, make_inputs, to_dev

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
    close(got, ref)


def test_rejects_problems_beyond_the_fixed_scratch():
    # 1M tokens x 32 heads needs a selection table far above the fixed array
    fake = 0x1000
    rc = moba.lib().moba_fwd_noalloc(fake, fake, fake, 1 << 20, 32, 8, 128, 4096, 12, fake, fake, None)
    assert rc == moba.MOBA_ERR_UNSUPPORTED
    assert "too large for moba_fwd_noalloc" in moba.last_error()
