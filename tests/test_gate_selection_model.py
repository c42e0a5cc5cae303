"""The gate kernel's selection scheme, modelled step by step on the CPU.

`gate_tc_kernel` (csrc/gate_tc.cuh) picks each row's best KP past blocks
without sorting all of them: a bound tau from the maxima of disjoint column
groups lets most columns skip the sorted insertion. The bound is only a
filter, so the result must be exactly the top KP by (score descending, block
ascending), the tie rule of the "How It Works" top-k gate. This module walks
the kernel's steps in plain Python (super-chunks of 128 columns, 32-column
pieces, group c mod NG, the KP-th largest maximum as tau, one compare per
column against max(tau, the float above the KP-th best), insertion in
ascending column order with a strictly-greater rule) in both modes the kernel
has: two passes (maxima over every super-chunk first) and one pass (the bound
grown super-chunk by super-chunk, later columns folded into the sorted
slots), and compares with brute force on scores full of ties.
"""
import numpy as np
import pytest

SC_COLS = 128
PIECE = 32


def groups_for(kp):
    # the kernel's GateCfg<KP>::kGroups; lists of more than 32 have no bound
    if kp > 32:
        return 0
    return 8 if kp <= 2 else (16 if kp <= 4 else 32)


def float_above(x):
    return np.nextafter(np.float32(x), np.float32(np.inf), dtype=np.float32)


def insert(tv, ti, s, j):
    # sorted descending; a block enters only with a strictly larger score
    kp = len(tv)
    for i in range(kp - 1, -1, -1):
        above = i > 0 and s > tv[i - 1]
        here = (not above) and s > tv[i]
        if above:
            tv[i], ti[i] = tv[i - 1], ti[i - 1]
        elif here:
            tv[i], ti[i] = s, j


def model_select(scores, kp, two_pass):
    scores = np.asarray(scores, dtype=np.float32)
    n = scores.size
    ng = groups_for(kp)
    nsc = (n + SC_COLS - 1) // SC_COLS
    tv = [np.float32(-np.inf)] * kp
    ti = [-1] * kp
    gm = [np.float32(-np.inf)] * max(ng, 1)
    tau = np.float32(-np.inf)
    two = ng > 0 and nsc > 1 and two_pass
    phases = [(sc, True) for sc in range(nsc)] + [(sc, False) for sc in range(nsc)] if two else \
        [(sc, None) for sc in range(nsc)]
    for sc, pass1_only in phases:
        cols = scores[sc * SC_COLS:(sc + 1) * SC_COLS]
        if ng > 0 and (pass1_only or not two):
            for e in range(cols.size):
                g = (e % PIECE) % ng  # the kernel indexes its slots by the column within the piece
                gm[g] = max(gm[g], cols[e])
            if not two or sc == nsc - 1:
                gm.sort(reverse=True)  # in place: later columns fold into the sorted slots
                tau = gm[kp - 1]
        if pass1_only:
            continue
        for p0 in range(0, cols.size, PIECE):
            lo = max(tau, float_above(tv[kp - 1]))
            for e in range(p0, min(p0 + PIECE, cols.size)):
                v = cols[e]
                if v >= lo and v > tv[kp - 1]:
                    insert(tv, ti, v, sc * SC_COLS + e)
    npast = min(kp, n)
    return sorted(ti[:npast])


def brute(scores, kp):
    scores = np.asarray(scores, dtype=np.float32)
    order = sorted(range(scores.size), key=lambda j: (-float(scores[j]), j))
    return sorted(order[:min(kp, scores.size)])


@pytest.mark.parametrize("kp", [2, 4, 8, 11, 12, 16, 24, 32, 48])
@pytest.mark.parametrize("n", [1, 5, 31, 32, 33, 127, 128, 129, 255, 300, 520])
def test_both_modes_give_the_exact_top_k_with_lowest_index_ties(kp, n):
    rng = np.random.default_rng(1000 * kp + n)
    for trial in range(12):
        if trial % 3 == 0:
            s = rng.standard_normal(n)                      # distinct scores
        elif trial % 3 == 1:
            s = rng.integers(-3, 4, size=n).astype(np.float64)  # heavy ties
        else:
            s = np.round(rng.standard_normal(n), 1)         # ties across groups and pieces
        s = s.astype(np.float32)
        want = brute(s, kp)
        assert model_select(s, kp, two_pass=True) == want
        assert model_select(s, kp, two_pass=False) == want


def test_a_bound_that_dropped_an_equal_score_would_be_caught():
    # plants the mistake the strict/non-strict split guards against: a
    # candidate test of v > tau (instead of v >= tau) loses a block whose
    # score equals the bound
    s = np.array([5, 5, 5, 1, 1, 1, 1, 1] * 8, dtype=np.float32)
    kp = 2
    ng = groups_for(kp)
    gm = sorted([max(s[g::ng]) for g in range(ng)], reverse=True)
    tau = gm[kp - 1]
    strict = [j for j in range(s.size) if s[j] > tau]
    assert len(strict) < kp          # the wrong test keeps too few
    assert model_select(s, kp, True) == brute(s, kp) == [0, 1]
