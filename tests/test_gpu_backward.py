"""The backward pass (moba_bwd) against the fp64 oracle of oracle/backward.py.

The GPU's selection is checked against the oracle gate first (as for the
forward) and then fixed for both sides, so the comparison is of the
gradients alone. Tolerance, from the arithmetic: P and dS enter the tensor
cores as bf16 (relative rounding 2^-9), D = rowsum(dO * O) uses the forward's
bf16 output, the dQ partials are fp16 and the outputs bf16; each gradient
element is a sum of many such terms, so the max-abs error is held to 2 % of
the largest reference magnitude and the mean-abs error to 1 % of the mean
reference magnitude, per tensor, plus an absolute floor for tensors that
are exactly zero (one token: P = 1 so dS = dP - D = 0): D from the bf16
output O differs from the exact one by about 2^-9 |dO||O|, which moves dQ by
at most ~1e-3 at these magnitudes.
"""
import numpy as np
import pytest

from parity_helpers import check_sel_structure, check_selection, make_inputs, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

import block_sparse_long_fwd_b200 as moba  # noqa: E402
import oracle  # noqa: E402
import synth_inputs as si  # noqa: E402
from oracle import backward as ob  # noqa: E402

MAX_REL = 2e-2
MEAN_REL = 1e-2
MAX_ABS_FLOOR = 1e-3
MEAN_ABS_FLOOR = 1e-4


def gpu_backward(q, k, v, do, B, topk):
    qd, kd, vd, dod = to_dev(q), to_dev(k), to_dev(v), to_dev(do)
    out, lse = moba.fwd(qd, kd, vd, B, topk)
    dq, dk, dv = moba.bwd(qd, kd, vd, out, lse, dod, B, topk)
    sel = moba.gate(qd, moba.pool(kd, B), k.shape[1], B, topk)
    torch.cuda.synchronize()
    assert moba.device_status() == moba.MOBA_OK
    f = lambda x: x.float().cpu().numpy().astype(np.float64)  # noqa: E731
    return f(dq), f(dk), f(dv), sel.cpu().numpy()


def compare(name, got, ref):
    err = np.abs(got - ref)
    stats = dict(max_err=float(err.max()), max_ref=float(np.abs(ref).max()), mean_err=float(err.mean()),
                 mean_ref=float(np.abs(ref).mean()))
    assert stats["max_err"] <= MAX_REL * stats["max_ref"] + MAX_ABS_FLOOR, (name, stats)
    assert stats["mean_err"] <= MEAN_REL * stats["mean_ref"] + MEAN_ABS_FLOOR, (name, stats)
    return stats


CASES = [
    # S,    Hq, Hkv, B,   topk, seed
    (1000,  4,  2,   256, 3,    1),   # GQA, ragged tail, routed blocks
    (1500,  2,  2,   256, 3,    2),   # one q head per kv head: paired own tiles
    (900,   2,  1,   128, 4,    3),   # 128-token blocks, two q heads per kv head
    (600,   2,  1,   256, 8,    4),   # topk >= blocks: the dense path
    (500,   2,  2,   128, 1,    5),   # own block only
    (1,     2,  1,   128, 3,    6),   # one token
    (4096,  4,  1,   512, 4,    7),   # 4K tokens, four q heads on one kv head, three routed blocks per row:
                                      # dK / dV summed over a group's heads and over routed and own rows
]


@pytest.mark.parametrize("S,Hq,Hkv,B,topk,seed", CASES)
def test_backward_matches_the_oracle(S, Hq, Hkv, B, topk, seed):
    w, q, k, v = make_inputs(S, Hq, Hkv, B, topk, 500 + seed)
    do = si.make_dout(w)
    dq, dk, dv, sel = gpu_backward(q, k, v, do, B, topk)
    check_sel_structure(sel, S, B, topk)
    rows_t, rows_h = oracle.all_rows(S, Hq)
    sel_acc, _ = check_selection(q, k, sel[rows_h, rows_t], rows_t, rows_h, B, Hkv, topk)
    sel_fixed = sel_acc.reshape(S, Hq, -1).transpose(1, 0, 2)
    rq, rk, rv, _, _ = ob.backward(q, k, v, do, B, topk, sel_fixed)
    compare("dq", dq, rq)
    compare("dk", dk, rk)
    compare("dv", dv, rv)


def test_backward_over_several_windows(monkeypatch):
    # query windows split the router lists and add dK / dV per window
    monkeypatch.setenv("MOBA_WINDOW", "256")
    S, Hq, Hkv, B, topk = 1200, 4, 2, 256, 3
    w, q, k, v = make_inputs(S, Hq, Hkv, B, topk, 77)
    do = si.make_dout(w)
    dq, dk, dv, sel = gpu_backward(q, k, v, do, B, topk)
    rows_t, rows_h = oracle.all_rows(S, Hq)
    sel_acc, _ = check_selection(q, k, sel[rows_h, rows_t], rows_t, rows_h, B, Hkv, topk)
    rq, rk, rv, _, _ = ob.backward(q, k, v, do, B, topk, sel_acc.reshape(S, Hq, -1).transpose(1, 0, 2))
    compare("dq", dq, rq)
    compare("dk", dk, rk)
    compare("dv", dv, rv)


def test_backward_is_deterministic():
    S, Hq, Hkv, B, topk = 3000, 4, 2, 256, 4
    w, q, k, v = make_inputs(S, Hq, Hkv, B, topk, 88)
    qd, kd, vd, dod = to_dev(q), to_dev(k), to_dev(v), to_dev(si.make_dout(w))
    out, lse = moba.fwd(qd, kd, vd, B, topk)
    a = moba.bwd(qd, kd, vd, out, lse, dod, B, topk)
    b = moba.bwd(qd, kd, vd, out, lse, dod, B, topk)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_backward_identities_and_sampled_rows_at_a_longer_shape():
    # 32K tokens, 8 q / 2 kv heads, 1024-token blocks, top-6: sum_s dK = 0
    # and sum_s dV = sum dO per kv head hold at any size; sampled dQ rows
    # against the oracle's single-row gradient
    S, Hq, Hkv, B, topk = 32768, 8, 2, 1024, 6
    w, q, k, v = make_inputs(S, Hq, Hkv, B, topk, 99)
    do = si.make_dout(w)
    dq, dk, dv, sel = gpu_backward(q, k, v, do, B, topk)
    G = Hq // Hkv
    # a sum of S random-sign terms is about sqrt(sum of squares); the
    # identities must cancel far below that (bf16 rounding leaves ~2^-9 of it)
    rms_k = np.sqrt((dk ** 2).sum(axis=0))
    assert np.all(np.abs(dk.sum(axis=0)) <= 0.05 * rms_k), np.abs(dk.sum(axis=0) / rms_k).max()
    want = ob.bf16_to_f64(do).reshape(S, Hkv, G, 128).sum(axis=(0, 2))
    rms_v = np.sqrt((dv ** 2).sum(axis=0))
    assert np.all(np.abs(dv.sum(axis=0) - want) <= 0.05 * rms_v), np.abs((dv.sum(axis=0) - want) / rms_v).max()
    rng = np.random.default_rng(5)
    rows_t = np.concatenate([[0, B - 1, B, S - 1], rng.integers(0, S, 28)])
    rows_h = rng.integers(0, Hq, rows_t.size)
    sel_rows, _ = check_selection(q, k, sel[rows_h, rows_t], rows_t, rows_h, B, Hkv, topk)
    ref = ob.dq_rows(q, k, v, do, B, rows_t, rows_h, sel_rows)
    compare("dq rows", dq[rows_t, rows_h], ref)
