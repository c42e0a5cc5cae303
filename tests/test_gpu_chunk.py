"""Chunked prefill and decode (moba_fwd_chunk) against the whole forward pass.

By causality, rows q_start..S-1 of the forward pass do not depend on the
queries of earlier tokens, and every row's arithmetic (gate scores, top-k,
online softmax, merge) is its own: so the chunk's output must equal those
rows of moba_fwd bit for bit, whatever other rows shared its tiles. One
decode row is also checked against the fp64 oracle.
"""
import numpy as np
import pytest

from parity_helpers import LSE_ABS, OUT_MAX_ABS, make_inputs, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

import block_sparse_long_fwd_b200 as moba  # noqa: E402
import oracle  # noqa: E402

CASES = [
    # S,   Hq, Hkv, B,   topk, q_start
    (3000, 4,  2,   256, 4,    1000),   # chunk starting inside a 128-token tile
    (3000, 4,  2,   256, 4,    2999),   # one decode step
    (4096, 2,  2,   512, 3,    2048),   # chunk at a block boundary, one head per group
    (4096, 1,  1,   512, 3,    3900),   # one head per group, inside a tile pair
    (5000, 8,  2,   512, 6,    4999),   # decode, four q heads per kv head
    (2000, 2,  1,   256, 64,   1500),   # topk >= blocks: the dense path
    (300,  2,  1,   128, 3,    0),      # q_start 0 is the whole forward
    # 320 past blocks (three 128-column super-chunks): the chunk's gate grid
    # fits one wave and takes the single pass, the whole forward's (1,282
    # CTAs) the two passes; the rows must still agree bit for bit
    (41000, 4, 2,   128, 12,   40999),
    (41000, 4, 2,   128, 12,   40700),
]


@pytest.mark.parametrize("S,Hq,Hkv,B,topk,q0", CASES)
def test_chunk_equals_rows_of_the_whole_forward(S, Hq, Hkv, B, topk, q0):
    _, q, k, v = make_inputs(S, Hq, Hkv, B, topk, 100 + q0 % 97)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    out, lse = moba.fwd(qd, kd, vd, B, topk)
    out_c, lse_c = moba.fwd_chunk(qd[q0:].contiguous(), kd, vd, B, topk)
    torch.cuda.synchronize()
    assert moba.device_status() == moba.MOBA_OK
    assert torch.equal(out_c, out[q0:])
    assert torch.equal(lse_c, lse[:, q0:])


def test_chunk_over_several_windows(monkeypatch):
    monkeypatch.setenv("MOBA_WINDOW", "512")
    S, Hq, Hkv, B, topk, q0 = 6000, 4, 2, 512, 5, 1234
    _, q, k, v = make_inputs(S, Hq, Hkv, B, topk, 55)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    out, lse = moba.fwd(qd, kd, vd, B, topk)
    out_c, lse_c = moba.fwd_chunk(qd[q0:].contiguous(), kd, vd, B, topk)
    torch.cuda.synchronize()
    assert torch.equal(out_c, out[q0:])
    assert torch.equal(lse_c, lse[:, q0:])


def test_decode_row_against_the_oracle():
    S, Hq, Hkv, B, topk = 8192, 8, 2, 512, 6
    _, q, k, v = make_inputs(S, Hq, Hkv, B, topk, 77)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    out_c, lse_c = moba.fwd_chunk(qd[S - 1:].contiguous(), kd, vd, B, topk)
    torch.cuda.synchronize()
    rows_t = np.full(Hq, S - 1, dtype=np.int64)
    rows_h = np.arange(Hq, dtype=np.int32)
    out_o, lse_o, _ = oracle.attend(q, k, v, B, topk, rows_t, rows_h)
    err = np.abs(out_c[0].float().cpu().numpy() - out_o).max()
    assert err <= OUT_MAX_ABS, err
    assert np.abs(lse_c[:, 0].cpu().numpy() - lse_o).max() <= LSE_ABS


@pytest.mark.parametrize("S,Hq,Hkv,B,topk,q0", [(5000, 8, 2, 512, 6, 4999), (3000, 4, 2, 256, 4, 1000)])
def test_chunk_with_the_callers_means(S, Hq, Hkv, B, topk, q0):
    # means from pool() replace the per-call pooling; they only steer the
    # gate, so the chunk's rows come out the same
    _, q, k, v = make_inputs(S, Hq, Hkv, B, topk, 300 + q0 % 89)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    qc = qd[q0:].contiguous()
    ref = moba.fwd_chunk(qc, kd, vd, B, topk)
    kmean = moba.pool(kd, B)
    got = moba.fwd_chunk(qc, kd, vd, B, topk, kmean=kmean)
    torch.cuda.synchronize()
    assert moba.device_status() == moba.MOBA_OK
    assert torch.equal(got[0], ref[0])
    assert torch.equal(got[1], ref[1])
