"""Pins for the backward oracle (oracle/backward.py), CPU only.

Each check compares it with something other than itself: torch autograd in
fp64 on the same masked attention (a library routine), exact identities of
the softmax gradient, linearity in the upstream gradient, and the C oracle's
forward values. A plausible slip (a dropped row-sum term, a sign, the scale
on the wrong factor, a transposed product, a head-group mix-up) fails one.
"""
import numpy as np
import pytest

import oracle
import synth_inputs as si
from oracle import backward as ob

torch = pytest.importorskip("torch")


def case(S, Hq, Hkv, B, topk, seed):
    w = si.Workload("bwd", S, Hq, Hkv, 128, B, topk, seed)
    q, k, v = si.make_qkv(w, threads=2)
    do = si.make_dout(w, threads=2)
    return q, k, v, do


CASES = [
    (300, 2, 1, 64, 3, 11),    # ragged tail, several routed blocks
    (256, 4, 2, 32, 4, 12),    # GQA: two q heads per kv head
    (200, 1, 1, 64, 8, 13),    # topk >= blocks: full causal attention
    (190, 2, 2, 128, 1, 14),   # topk 1: own block only
]


def autograd_reference(q, k, v, do, B, sel):
    """torch fp64 autograd through softmax(c Q K^T + mask) V with the same row masks."""
    Q, K, V, dO = (torch.tensor(ob.bf16_to_f64(x), requires_grad=True) for x in (q, k, v, do))
    S, Hq, d = Q.shape
    G = Hq // K.shape[1]
    outs = []
    for h in range(Hq):
        g = h // G
        M = torch.tensor(ob.row_mask(sel[h], S, B))
        logits = (Q[:, h] @ K[:, g].T) / d ** 0.5
        logits = logits.masked_fill(~M, float("-inf"))
        outs.append(torch.softmax(logits, dim=1) @ V[:, g])
    out = torch.stack(outs, dim=1)
    (out * dO.detach()).sum().backward()
    return Q.grad.numpy(), K.grad.numpy(), V.grad.numpy(), out.detach().numpy()


@pytest.mark.parametrize("S,Hq,Hkv,B,topk,seed", CASES)
def test_matches_torch_autograd(S, Hq, Hkv, B, topk, seed):
    q, k, v, do = case(S, Hq, Hkv, B, topk, seed)
    sel = ob.full_selection(q, k, B, topk)
    dq, dk, dv, out, _ = ob.backward(q, k, v, do, B, topk, sel)
    rq, rk, rv, rout = autograd_reference(q, k, v, do, B, sel)
    for a, b in ((dq, rq), (dk, rk), (dv, rv), (out, rout)):
        np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-11)


@pytest.mark.parametrize("S,Hq,Hkv,B,topk,seed", CASES)
def test_gradient_identities(S, Hq, Hkv, B, topk, seed):
    # each row of dS sums to zero (softmax rows sum to one), so the keys' dK
    # sum to zero per kv head; the rows of P sum to one, so the keys' dV sum
    # to the group's upstream gradients
    q, k, v, do = case(S, Hq, Hkv, B, topk, seed)
    dq, dk, dv, _, _ = ob.backward(q, k, v, do, B, topk)
    G = Hq // Hkv
    dO = ob.bf16_to_f64(do)
    scale = np.abs(dk).max()
    assert np.abs(dk.sum(axis=0)).max() <= 1e-10 * scale * S
    want = dO.reshape(S, Hkv, G, 128).sum(axis=(0, 2))
    np.testing.assert_allclose(dv.sum(axis=0), want, rtol=1e-10, atol=1e-9)


def test_linear_in_the_upstream_gradient():
    q, k, v, do = case(260, 2, 1, 64, 3, 21)
    _, _, _, do2 = case(260, 2, 1, 64, 3, 22)
    sel = ob.full_selection(q, k, 64, 3)
    a = ob.backward(q, k, v, do, 64, 3, sel)
    b = ob.backward(q, k, v, do2, 64, 3, sel)
    # dO1 + dO2 in fp64 is not a bf16 input; compare the sum through the
    # autograd reference, which takes any dO
    Q, K, V = (torch.tensor(ob.bf16_to_f64(x), requires_grad=True) for x in (q, k, v))
    dsum = torch.tensor(ob.bf16_to_f64(do) + ob.bf16_to_f64(do2))
    outs = []
    for h in range(2):
        M = torch.tensor(ob.row_mask(sel[h], 260, 64))
        logits = ((Q[:, h] @ K[:, 0].T) / 128 ** 0.5).masked_fill(~M, float("-inf"))
        outs.append(torch.softmax(logits, dim=1) @ V[:, 0])
    (torch.stack(outs, dim=1) * dsum).sum().backward()
    for i, g in enumerate((Q.grad, K.grad, V.grad)):
        np.testing.assert_allclose(a[i] + b[i], g.numpy(), rtol=1e-9, atol=1e-11)


def test_forward_values_match_the_c_oracle():
    q, k, v, do = case(300, 4, 2, 64, 3, 31)
    _, _, _, out, lse = ob.backward(q, k, v, do, 64, 3)
    out_c, lse_c, _ = oracle.attend(q, k, v, 64, 3)
    S, Hq = 300, 4
    np.testing.assert_allclose(out.reshape(S * Hq, 128), out_c, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.T.reshape(-1), lse_c, rtol=0, atol=1e-12)


def test_single_row_dq_matches_the_dense_version():
    q, k, v, do = case(300, 4, 2, 64, 3, 41)
    sel = ob.full_selection(q, k, 64, 3)
    dq = ob.backward(q, k, v, do, 64, 3, sel)[0]
    rows_t = np.array([0, 63, 64, 150, 299, 299])
    rows_h = np.array([0, 1, 2, 3, 0, 3])
    got = ob.dq_rows(q, k, v, do, 64, rows_t, rows_h, sel[rows_h, rows_t])
    np.testing.assert_allclose(got, dq[rows_t, rows_h], rtol=1e-10, atol=1e-12)


def test_a_planted_mistake_is_caught():
    # dropping the softmax Jacobian's row-sum term breaks the dK identity
    q, k, v, do = case(256, 2, 1, 64, 3, 51)
    sel = ob.full_selection(q, k, 64, 3)
    Q, K, V, dO = (ob.bf16_to_f64(x) for x in (q, k, v, do))
    M = ob.row_mask(sel[0], 256, 64)
    logits = np.where(M, (Q[:, 0] @ K[:, 0].T) / np.sqrt(128), -np.inf)
    P = np.exp(logits - logits.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    wrong_dS = P * (dO[:, 0] @ V[:, 0].T)  # the D term left out
    wrong_dk = (wrong_dS.T @ Q[:, 0]) / np.sqrt(128)
    assert np.abs(wrong_dk.sum(axis=0)).max() > 1e-3
