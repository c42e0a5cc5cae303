"""The router's flag-word walk, modelled on the CPU.

`route_flags_kernel` (csrc/route.cuh) writes, for one warp's 32 group-rows,
flag word bits[j] (bit l set when row l routes to past block j) for every
block some row picked, into words cleared beforehand. Instead of a pass over
every past block it repeats: j = the smallest entry still pending in any lane
(a warp minimum), the lanes holding j set their bit and advance. This is the
MoE-style dispatch of the "How It Works" routing: each row's chosen past
blocks become its membership in per-block lists. The walk relies on each row's
past entries being ascending and below its own block; the model checks that
it reproduces the dense construction, and that it visits exactly the distinct
picked blocks.
"""
import numpy as np
import pytest

INF = 0x7FFFFFFF


def dense_words(rows, bts, nblocks):
    words = np.zeros(nblocks, dtype=np.uint64)
    for lane, (sel, bt) in enumerate(zip(rows, bts)):
        for j in sel:
            if 0 <= j < bt:
                words[j] |= np.uint64(1) << np.uint64(lane)
    return words


def walk_words(rows, bts, nblocks):
    words = np.zeros(nblocks, dtype=np.uint64)  # cleared before the walk
    entries = [[j if 0 <= j < bt else INF for j in sel] for sel, bt in zip(rows, bts)]
    ptr = [0] * len(rows)
    cur = [e[0] if e else INF for e in entries]
    steps = 0
    while True:
        j = min(cur)                      # the warp minimum
        if j == INF:
            break
        bits = 0
        for lane in range(len(rows)):
            if cur[lane] == j:            # the lanes that picked j
                bits |= 1 << lane
                ptr[lane] += 1
                cur[lane] = entries[lane][ptr[lane]] if ptr[lane] < len(entries[lane]) else INF
        words[j] = np.uint64(bits)        # lane 0's store
        steps += 1
    return words, steps


@pytest.mark.parametrize("nblocks,p", [(4, 1), (16, 3), (64, 11), (256, 11), (300, 47)])
def test_the_walk_writes_the_dense_flag_words(nblocks, p):
    rng = np.random.default_rng(nblocks * 100 + p)
    for _ in range(40):
        rows, bts = [], []
        for _lane in range(32):
            bt = int(rng.integers(0, nblocks + 1))          # the row's own block
            npast = min(p, bt)
            past = sorted(rng.choice(bt, size=npast, replace=False).tolist()) if npast else []
            sel = past + [bt] + [-1] * (p - npast)          # the gate's row layout (own block, then padding)
            rows.append(sel[:p])                            # the walk reads the first k - 1 entries
            bts.append(bt)
        want = dense_words(rows, bts, nblocks + 1)
        got, steps = walk_words(rows, bts, nblocks + 1)
        assert np.array_equal(got, want)
        assert steps == int(np.count_nonzero(want))         # one step per distinct picked block


def test_an_unsorted_row_would_be_caught():
    # a row whose entries were not ascending revisits a block after its word
    # was written and overwrites another row's bit: the model shows what the
    # ascending order of the gate's output guarantees
    rows = [[5, 2], [2]] + [[] for _ in range(30)]
    bts = [9, 9] + [0] * 30
    got, _ = walk_words(rows, bts, 10)
    want = dense_words(rows, bts, 10)
    assert want[2] == 3 and got[2] == 1
