"""Pins for the fp64 oracle, each against something other than the oracle.

Every check here fixes part of the oracle to a closed form, a library
routine (torch's scaled-dot-product attention, logsumexp, numpy matmul/mean),
brute force on tiny inputs, or an invariant that the method's definition
implies:

- mean-pool: integer-valued keys whose block means have a closed form;
- gate + top-k: exhaustive search over all (k-1)-subsets of past blocks on
  integer scores with planted ties (lowest index wins);
- full mode: topk >= number of blocks is dense causal attention (the pages:
  seamless switch between full and sparse attention);
- topk = 1 is causal attention inside each block on its own;
- general masks: torch attention under a boolean mask built from the brute
  force selection;
- invariants: constant V, GQA vs repeated KV heads, prefix invariance
  (causality), LSE non-decreasing in topk, outputs inside the hull of V.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle


def bf16(x) -> np.ndarray:
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def f64(u: np.ndarray) -> np.ndarray:
    return (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rand_qkv(S, Hq, Hkv, d, seed, scale=1.0):
    g = np.random.default_rng(seed)
    q = bf16(g.standard_normal((S, Hq, d)) * scale)
    k = bf16(g.standard_normal((S, Hkv, d)) * scale)
    v = bf16(g.standard_normal((S, Hkv, d)))
    return q, k, v


def torch_masked_attention(q, k, v, mask_fn):
    """out, lse via torch library routines: SDPA with a boolean mask, logsumexp."""
    S, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    Q = torch.from_numpy(f64(q)).permute(1, 0, 2)  # [Hq][S][d]
    K = torch.from_numpy(f64(k)).permute(1, 0, 2).repeat_interleave(G, dim=0)
    V = torch.from_numpy(f64(v)).permute(1, 0, 2).repeat_interleave(G, dim=0)
    mask = torch.zeros(Hq, S, S, dtype=torch.bool)
    for h in range(Hq):
        for t in range(S):
            mask[h, t] = torch.from_numpy(mask_fn(t, h))
    out = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask)
    logits = (Q @ K.transpose(1, 2)) / np.sqrt(d)
    lse = torch.logsumexp(logits.masked_fill(~mask, -np.inf), dim=-1)
    return out.permute(1, 0, 2).numpy(), lse.numpy()  # [S][Hq][d], [Hq][S]


def as_rows(out, lse, S, Hq):
    """oracle row order is t-major: reshape to [S][Hq][d] and [Hq][S]."""
    return out.reshape(S, Hq, -1), lse.reshape(S, Hq).T


# ---------------------------------------------------------------- mean-pool

@pytest.mark.parametrize("S,B", [(64, 16), (70, 16), (8, 8), (5, 8)])
def test_kmean_closed_form(S, B):
    Hkv, d = 2, 4
    # K[t][g][c] = t + c + 3g: integers < 256, exact in bf16
    k = np.empty((S, Hkv, d), dtype=np.float64)
    for t in range(S):
        for g in range(Hkv):
            for c in range(d):
                k[t, g, c] = t + c + 3 * g
    m = oracle.kmean(bf16(k), B)
    nb = (S + B - 1) // B
    for g in range(Hkv):
        for j in range(nb):
            t0, t1 = j * B, min(S, (j + 1) * B) - 1
            for c in range(d):
                # arithmetic series: mean of t over [t0, t1] is (t0 + t1) / 2
                assert m[g, j, c] == (t0 + t1) / 2 + c + 3 * g


# ------------------------------------------------------------- gate + top-k

def brute_force_sel(scores, b, k_eff):
    """Max-sum (k-1)-subset of past blocks; lexicographically first among ties."""
    npast = min(k_eff - 1, b)
    best, best_tot = None, None
    for comb in itertools.combinations(range(b), npast):
        tot = sum(scores[j] for j in comb)
        if best is None or tot > best_tot:
            best, best_tot = comb, tot
    return sorted(best) + [b]


@pytest.mark.parametrize("topk", [1, 2, 3, 4, 6, 9])
@pytest.mark.parametrize("Hq,Hkv", [(1, 1), (4, 2)])
def test_select_brute_force_with_ties(topk, Hq, Hkv):
    S, B, d = 64, 8, 4
    nb = S // B
    rng = np.random.default_rng(100 + topk)
    # every key of block j of head g equals a small integer vector, drawn from
    # only three choices so that many scores tie exactly
    choices = np.array([[1, 0, -1, 2], [0, 1, 1, 0], [1, 0, -1, 2]], dtype=np.float64)
    k = np.empty((S, Hkv, d))
    for g in range(Hkv):
        for j in range(nb):
            k[j * B:(j + 1) * B, g] = choices[rng.integers(0, 3)]
    q = rng.integers(-2, 3, size=(S, Hq, d)).astype(np.float64)
    kb, qb = bf16(k), bf16(q)
    m = oracle.kmean(kb, B)
    # library routines for the scores: numpy mean and matmul
    m_np = f64(kb).reshape(nb, B, Hkv, d).mean(axis=1)  # [nb][Hkv][d]
    rows_t, rows_h = oracle.all_rows(S, Hq)
    sel, info = oracle.select(qb, m, B, Hkv, topk, rows_t, rows_h)
    k_eff = min(topk, nb)
    G = Hq // Hkv
    for r, (t, h) in enumerate(zip(rows_t, rows_h)):
        b = t // B
        scores = f64(qb)[t, h] @ m_np[:b, h // G].T if b else np.zeros(0)
        want = brute_force_sel(scores, b, k_eff)
        got = [x for x in sel[r] if x >= 0]
        assert got == want, (t, h, scores, got, want)
        assert list(sel[r][len(want):]) == [-1] * (k_eff - len(want))


def test_gate_scores_library_matmul():
    S, Hq, Hkv, d, B = 96, 4, 2, 8, 16
    q, k, _ = rand_qkv(S, Hq, Hkv, d, 3)
    m = oracle.kmean(k, B)
    for t, h in [(95, 3), (40, 0), (16, 1), (15, 2)]:
        s = oracle.gate_scores(q, m, B, Hkv, t, h)
        ref = f64(q)[t, h] @ m[h // (Hq // Hkv), : t // B].T
        assert s.shape == (t // B,)
        np.testing.assert_allclose(s, ref, rtol=1e-13, atol=1e-13)


def test_select_gap_info():
    S, Hq, Hkv, d, B = 128, 2, 1, 8, 16
    q, k, _ = rand_qkv(S, Hq, Hkv, d, 5)
    m = oracle.kmean(k, B)
    rows_t, rows_h = oracle.all_rows(S, Hq)
    sel, info = oracle.select(q, m, B, Hkv, 3, rows_t, rows_h)
    for r, (t, h) in enumerate(zip(rows_t, rows_h)):
        b = t // B
        raw = f64(q)[t, h] @ m[0, :b].T
        s = np.sort(raw)[::-1]
        scale = np.abs(raw).max() if b else 0.0
        assert info[r, 3] == pytest.approx(scale, rel=1e-12, abs=1e-300)
        if 1 <= 2 < b:
            sa, sb = s[1], s[2]
            assert info[r, 1] == pytest.approx(sa, rel=1e-12)
            assert info[r, 2] == pytest.approx(sb, rel=1e-12)
            assert info[r, 0] == pytest.approx((sa - sb) / scale, rel=1e-9, abs=1e-15)
        else:
            assert np.isinf(info[r, 0])


# ------------------------------------------------------------ attention

@pytest.mark.parametrize("S,B,Hq,Hkv", [(64, 8, 1, 1), (60, 16, 4, 2), (33, 8, 2, 1)])
def test_full_mode_is_causal_attention(S, B, Hq, Hkv):
    d = 8
    q, k, v = rand_qkv(S, Hq, Hkv, d, 7)
    nb = (S + B - 1) // B
    out, lse, sel = oracle.attend(q, k, v, B, topk=nb + 3)
    o, l = as_rows(out, lse, S, Hq)
    ref_o, ref_l = torch_masked_attention(q, k, v, lambda t, h: np.arange(S) <= t)
    np.testing.assert_allclose(o, ref_o, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(l, ref_l, rtol=1e-12, atol=1e-12)
    # also the library's own causal path
    G = Hq // Hkv
    Q = torch.from_numpy(f64(q)).permute(1, 0, 2)
    K = torch.from_numpy(f64(k)).permute(1, 0, 2).repeat_interleave(G, 0)
    V = torch.from_numpy(f64(v)).permute(1, 0, 2).repeat_interleave(G, 0)
    ref2 = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True).permute(1, 0, 2).numpy()
    np.testing.assert_allclose(o, ref2, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("S,B", [(64, 8), (50, 16), (7, 8)])
def test_topk1_is_blockwise_causal(S, B):
    Hq, Hkv, d = 2, 1, 8
    q, k, v = rand_qkv(S, Hq, Hkv, d, 9)
    out, lse, sel = oracle.attend(q, k, v, B, topk=1)
    o, l = as_rows(out, lse, S, Hq)
    Q = torch.from_numpy(f64(q)).permute(1, 0, 2)
    K = torch.from_numpy(f64(k)).permute(1, 0, 2).repeat_interleave(Hq, 0)
    V = torch.from_numpy(f64(v)).permute(1, 0, 2).repeat_interleave(Hq, 0)
    ref = np.empty_like(o)
    for j in range(0, S, B):
        e = min(S, j + B)
        blk = torch.nn.functional.scaled_dot_product_attention(Q[:, j:e], K[:, j:e], V[:, j:e], is_causal=True)
        ref[j:e] = blk.permute(1, 0, 2).numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-10, atol=1e-12)
    assert np.all(sel[:, 0] == oracle.all_rows(S, Hq)[0] // B)


@pytest.mark.parametrize("topk", [2, 3, 5])
def test_masked_attention_matches_library_under_brute_force_mask(topk):
    S, B, Hq, Hkv, d = 48, 8, 4, 2, 8
    q, k, v = rand_qkv(S, Hq, Hkv, d, 11 + topk)
    nb = S // B
    G = Hq // Hkv
    m_np = f64(k).reshape(nb, B, Hkv, d).mean(axis=1)
    sels = {}
    for t in range(S):
        for h in range(Hq):
            b = t // B
            s = f64(q)[t, h] @ m_np[:b, h // G].T if b else np.zeros(0)
            sels[(t, h)] = brute_force_sel(s, b, min(topk, nb))

    def mask_fn(t, h):
        u = np.arange(S)
        return np.isin(u // B, sels[(t, h)]) & (u <= t)

    out, lse, sel = oracle.attend(q, k, v, B, topk)
    o, l = as_rows(out, lse, S, Hq)
    ref_o, ref_l = torch_masked_attention(q, k, v, mask_fn)
    np.testing.assert_allclose(o, ref_o, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(l, ref_l, rtol=1e-12, atol=1e-12)


def test_constant_v_gives_constant_output():
    S, B, Hq, Hkv, d = 64, 8, 2, 1, 8
    q, k, _ = rand_qkv(S, Hq, Hkv, d, 13)
    c = np.linspace(-2, 2, d)
    v = bf16(np.broadcast_to(c, (S, Hkv, d)))
    out, _, _ = oracle.attend(q, k, v, B, 3)
    np.testing.assert_allclose(out, np.broadcast_to(f64(v)[0, 0], out.shape), rtol=1e-12, atol=1e-12)


def test_gqa_equals_mha_with_repeated_kv():
    S, B, Hq, Hkv, d = 64, 8, 4, 2, 8
    q, k, v = rand_qkv(S, Hq, Hkv, d, 17)
    G = Hq // Hkv
    out_g, lse_g, sel_g = oracle.attend(q, k, v, B, 3)
    k_rep = np.ascontiguousarray(np.repeat(k, G, axis=1))
    v_rep = np.ascontiguousarray(np.repeat(v, G, axis=1))
    out_m, lse_m, sel_m = oracle.attend(q, k_rep, v_rep, B, 3)
    assert np.array_equal(sel_g, sel_m)
    np.testing.assert_array_equal(out_g, out_m)
    np.testing.assert_array_equal(lse_g, lse_m)


def test_prefix_invariance():
    S, B, Hq, Hkv, d, P = 96, 8, 2, 1, 8, 40
    q, k, v = rand_qkv(S, Hq, Hkv, d, 19)
    out_f, lse_f, sel_f = oracle.attend(q, k, v, B, 3)
    out_p, lse_p, sel_p = oracle.attend(q[:P].copy(), k[:P].copy(), v[:P].copy(), B, 3)
    n = P * Hq
    assert np.array_equal(sel_f[:n], sel_p)
    np.testing.assert_array_equal(out_f[:n], out_p)
    np.testing.assert_array_equal(lse_f[:n], lse_p)


def test_lse_non_decreasing_in_topk_and_nested_selection():
    S, B, Hq, Hkv, d = 80, 8, 2, 1, 8
    q, k, v = rand_qkv(S, Hq, Hkv, d, 23)
    prev_lse, prev_sel = None, None
    for topk in range(1, 11):
        _, lse, sel = oracle.attend(q, k, v, B, topk)
        if prev_lse is not None:
            assert np.all(lse >= prev_lse - 1e-12)
            for r in range(sel.shape[0]):
                assert set(prev_sel[r][prev_sel[r] >= 0]) <= set(sel[r][sel[r] >= 0])
        prev_lse, prev_sel = lse, sel


def test_output_inside_hull_of_selected_values():
    S, B, Hq, Hkv, d = 64, 8, 1, 1, 8
    q, k, v = rand_qkv(S, Hq, Hkv, d, 29)
    out, _, sel = oracle.attend(q, k, v, B, 3)
    vf = f64(v)[:, 0]
    for t in range(S):
        keys = [u for u in range(t + 1) if (u // B) in set(sel[t])]
        lo, hi = vf[keys].min(axis=0), vf[keys].max(axis=0)
        assert np.all(out[t] >= lo - 1e-12) and np.all(out[t] <= hi + 1e-12)


def test_sel_override_and_row_subset():
    S, B, Hq, Hkv, d = 64, 8, 2, 2, 8
    q, k, v = rand_qkv(S, Hq, Hkv, d, 31)
    out_all, lse_all, sel_all = oracle.attend(q, k, v, B, 3)
    rows_t = np.array([63, 5, 40, 17], dtype=np.int64)
    rows_h = np.array([1, 0, 1, 0], dtype=np.int32)
    idx = rows_t * Hq + rows_h
    out_s, lse_s, sel_s = oracle.attend(q, k, v, B, 3, rows_t, rows_h)
    np.testing.assert_array_equal(out_s, out_all[idx])
    out_o, lse_o, _ = oracle.attend(q, k, v, B, 3, rows_t, rows_h, sel=sel_all[idx])
    np.testing.assert_array_equal(out_o, out_all[idx])
