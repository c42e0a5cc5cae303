"""GPU gate on exact ties: the lowest block index must win.

The gate's tie rule (equal scores go to the lower block index) cannot be
seen on the random workloads, where a tie is an accident and the selection
comparison allows near-ties either way. These inputs plant exact ties: every
block's keys are one of two or three small-integer vectors plus +-1/2 offsets
that cancel in pairs of tokens, so every block mean is exactly that integer
vector, and the queries are small integers. The gate scores are then small
integers on both sides (fp64 oracle; fp32 tensor-core sums of bf16 hi/lo
parts on the GPU, where lo = 0), many rows hold equal scores for several
past blocks, and the GPU selection must equal the oracle's on every row, bit
for bit. Lists of 2 to 64 entries are covered, including the 8- to 24-entry
lists whose first 64-block chunk is pre-filtered, and tables of up to 200
blocks (four chunks), so ties also fall across chunk boundaries.
"""
import numpy as np
import pytest

import oracle
from parity_helpers import bf16_bits, check_sel_structure, compare_outputs, run_gpu

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)


def planted_ties(S, Hq, Hkv, B, ntypes, seed):
    rng = np.random.default_rng(seed)
    nb = (S + B - 1) // B
    types = rng.integers(-1, 2, size=(Hkv, ntypes, 128)).astype(np.float32)
    which = rng.integers(0, ntypes, size=(Hkv, nb))
    blk = np.arange(S) // B
    k = types[np.arange(Hkv)[None, :], which[:, blk].T]  # [S][Hkv][128]
    # +-1/2 offsets that cancel over each pair of tokens (2i, 2i+1) of a block
    sign = rng.choice(np.array([-0.5, 0.5], dtype=np.float32), size=((S + 1) // 2, Hkv, 128))
    off = np.repeat(sign, 2, axis=0)[:S]
    off[1::2] *= -1.0
    k = k + off
    q = rng.integers(-1, 2, size=(S, Hq, 128)).astype(np.float32)
    v = rng.normal(0.0, 1.0, size=(S, Hkv, 128)).astype(np.float32)
    return bf16_bits(q), bf16_bits(k), bf16_bits(v)


CASES = [
    # S,     Hq, Hkv, B,   topk, types, seed
    (25600,  2,  1,   128, 9,    3,     1),   # 8-entry lists (first chunk pre-filtered), 200 blocks
    (25600,  4,  2,   128, 13,   2,     2),   # 12-entry lists, GQA, two key types: ties everywhere
    (12800,  2,  2,   128, 3,    3,     3),   # 2-entry lists
    (25600,  2,  1,   128, 25,   3,     4),   # 24-entry lists
    (12800,  1,  1,   128, 41,   2,     5),   # 48-entry lists
    (25600,  1,  1,   128, 65,   3,     6),   # 64-entry lists
    (9000,   2,  1,   384, 17,   3,     7),   # 16-entry lists, block 384, ragged tail
]


@pytest.mark.parametrize("S,Hq,Hkv,B,topk,ntypes,seed", CASES)
def test_exact_ties_go_to_the_lowest_block(S, Hq, Hkv, B, topk, ntypes, seed):
    q, k, v = planted_ties(S, Hq, Hkv, B, ntypes, seed)
    out_g, lse_g, sel_g, kmean_g = run_gpu(q, k, v, B, topk)
    m = oracle.kmean(k, B)
    nbp = oracle.nblocks(S, B) - 1
    # the planted means are exact integers, and so are the GPU's
    assert np.array_equal(kmean_g.astype(np.float64), m[:, :nbp])
    assert np.array_equal(m[:, :nbp], np.round(m[:, :nbp]))
    check_sel_structure(sel_g, S, B, topk)
    rows_t, rows_h = oracle.all_rows(S, Hq)
    sel_o, info = oracle.select(q, m, B, Hkv, topk, rows_t, rows_h)
    ties = int(np.sum(info[:, 0] == 0.0))
    assert ties > S * Hq // 10, ties  # the inputs really tie at the cut on many rows
    got = sel_g[rows_h, rows_t]
    bad = np.nonzero(np.any(got != sel_o, axis=1))[0]
    assert bad.size == 0, (f"{bad.size} rows differ; first t={rows_t[bad[0]]} h={rows_h[bad[0]]}: "
                           f"gpu {got[bad[0]]} oracle {sel_o[bad[0]]}")
    out_o, lse_o, _ = oracle.attend(q, k, v, B, topk, rows_t, rows_h, sel=sel_o)
    out_rows = out_g[torch.from_numpy(rows_t), torch.from_numpy(rows_h.astype(np.int64))].float().numpy()
    stats = compare_outputs(out_rows, lse_g[rows_h, rows_t], out_o, lse_o)
    print(dict(stats, tied_rows=ties))
