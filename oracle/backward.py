"""fp64 CPU oracle for the gradient of the MoBA forward pass (dQ, dK, dV).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: the tests,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs use it; the product
path never imports it.

What it computes. The pages ask for MoBA to be trained further from a full
attention model ("MoBA (Mixture of Block Attention)" project summary, "Key
Features" and "Limitations"; "Efficient Long-Context Attention with MoBA",
"How MoBA Works"), which needs the gradient of the forward pass. The gate's
top-k choice is piecewise constant in its inputs, so the gradient is taken
with the selection held fixed: each query row is ordinary causal softmax
attention over the keys of its selected blocks, and the block means, which
only steer the choice, receive no gradient. For one q head h of kv head g,
with scale c = 1/sqrt(d), the row mask M (selected past blocks plus the
causal part of the own block), P = softmax(c Q K^T) over M, O = P V and an
upstream gradient dO:

    dV   = sum over the group's q heads of P^T dO
    dP   = dO V^T
    dS   = P * (dP - rowsum(dO * O))
    dQ   = c dS K
    dK   = sum over the group's q heads of c dS^T Q

(the last two lines are the chain rule through the logits c Q K^T; the
row-sum term is the softmax Jacobian). The code below is that definition
written out with dense fp64 matrices per q head; it takes the selection as an
input (by default the oracle's own gate, ``oracle.select``).

Pins (tests/test_oracle_backward.py): torch autograd in fp64 on the same masked
attention; the exact identities sum_s dK[s][g] = 0 and
sum_s dV[s][g] = sum over (t, h in g) of dO[t][h]; linearity in dO; and the
forward values (out, lse) against the C oracle's ``attend``.
"""
from __future__ import annotations

import numpy as np

from . import all_rows, kmean, nblocks, select


def bf16_to_f64(a: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16 / int16 views) to fp64 values."""
    u = np.ascontiguousarray(a).view(np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def full_selection(q: np.ndarray, k: np.ndarray, block_size: int, topk: int) -> np.ndarray:
    """The oracle gate's choice for every row: int32 [Hq][S][k_eff]."""
    S, Hq, _ = q.shape
    Hkv = k.shape[1]
    rt, rh = all_rows(S, Hq)
    sel, _ = select(q, kmean(k, block_size), block_size, Hkv, topk, rt, rh)
    k_eff = sel.shape[1]
    return sel.reshape(S, Hq, k_eff).transpose(1, 0, 2).copy()


def row_mask(sel_h: np.ndarray, S: int, block_size: int) -> np.ndarray:
    """bool [S][S]: key s is attended by query t of this head."""
    t = np.arange(S)
    blk = t // block_size
    chosen = np.zeros((S, nblocks(S, block_size)), dtype=bool)
    for i in range(sel_h.shape[1]):
        j = sel_h[:, i]
        ok = j >= 0
        chosen[t[ok], j[ok]] = True
    chosen[t, blk] = True  # the own block is always attended
    return chosen[:, blk] & (t[None, :] <= t[:, None])


def backward(q, k, v, dout, block_size: int, topk: int, sel: np.ndarray | None = None):
    """Returns (dq [S][Hq][d], dk [S][Hkv][d], dv [S][Hkv][d], out, lse [Hq][S]), all fp64.

    q, k, v, dout: bf16 bit patterns [S][H][d]. ``sel`` [Hq][S][k_eff] (int32,
    -1 padded) fixes the selection; by default the oracle gate's.
    """
    Q, K, V, dO = (bf16_to_f64(x) for x in (q, k, v, dout))
    S, Hq, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    c = 1.0 / np.sqrt(d)
    if sel is None:
        sel = full_selection(q, k, block_size, topk)
    dq = np.zeros_like(Q)
    dk = np.zeros_like(K)
    dv = np.zeros_like(V)
    out = np.zeros_like(Q)
    lse = np.zeros((Hq, S))
    for h in range(Hq):
        g = h // G
        M = row_mask(sel[h], S, block_size)
        logits = np.where(M, c * (Q[:, h] @ K[:, g].T), -np.inf)
        mx = logits.max(axis=1, keepdims=True)
        e = np.exp(logits - mx)
        z = e.sum(axis=1, keepdims=True)
        P = e / z
        lse[h] = (mx + np.log(z))[:, 0]
        O = P @ V[:, g]
        out[:, h] = O
        dv[:, g] += P.T @ dO[:, h]
        dP = dO[:, h] @ V[:, g].T
        Drow = (dO[:, h] * O).sum(axis=1, keepdims=True)
        dS = P * (dP - Drow)
        dq[:, h] = c * (dS @ K[:, g])
        dk[:, g] += c * (dS.T @ Q[:, h])
    return dq, dk, dv, out, lse


def dq_rows(q, k, v, dout, block_size: int, rows_t, rows_h, sel_rows: np.ndarray):
    """dQ of single rows (t, h) with their selections sel_rows [n][k_eff]: the
    same definition restricted to one query, for sampled checks at sizes the
    dense version cannot hold. Returns fp64 [n][d]."""
    d = q.shape[2]
    G = q.shape[1] // k.shape[1]
    c = 1.0 / np.sqrt(d)
    res = np.zeros((len(rows_t), d))
    for n, (t, h) in enumerate(zip(rows_t, rows_h)):
        t, h = int(t), int(h)
        g = h // G
        bt = t // block_size
        blocks = sorted({int(j) for j in sel_rows[n] if 0 <= j < bt} | {bt})
        keys = np.concatenate([np.arange(j * block_size, min((j + 1) * block_size, t + 1)) for j in blocks])
        qv = bf16_to_f64(q[t, h])
        Kb = bf16_to_f64(k[keys, g])
        Vb = bf16_to_f64(v[keys, g])
        go = bf16_to_f64(dout[t, h])
        s = c * (Kb @ qv)
        p = np.exp(s - s.max())
        p /= p.sum()
        o = p @ Vb
        dp = Vb @ go
        ds = p * (dp - go @ o)
        res[n] = c * (ds @ Kb)
    return res
