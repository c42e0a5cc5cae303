"""Packed batches of independent sequences (moba_fwd_varlen).

Each sequence of a batch is its own causal MoBA problem (blocks start at its
first token, no attention across sequences), so its rows must equal moba_fwd
on its tokens alone bit for bit, and match the fp64 oracle run on that
sequence.
"""
import numpy as np
import pytest

from parity_helpers import full_check, make_inputs, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

import block_sparse_long_fwd_b200 as moba  # noqa: E402


def packed(lengths, Hq, Hkv, B, topk, seed):
    """Host inputs of each sequence (its own seeded synthetic workload) and
    the packed device tensors with their offsets."""
    seqs = [make_inputs(L, Hq, Hkv, B, topk, seed + i)[1:] if L else None for i, L in enumerate(lengths)]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    cat = [np.concatenate([s[j] for s in seqs if s is not None]) for j in range(3)]
    return seqs, cu, [to_dev(a) for a in cat]


CASES = [
    # lengths,                          Hq, Hkv, B,   topk
    ([3000, 0, 1, 4096, 777, 513],      4,  2,   256, 4),   # empty, one token, dense (nb <= topk) sequences
    ([1500, 2100, 129],                 2,  2,   512, 3),   # one q head per kv head (paired own tiles)
    ([5000, 4999],                      8,  2,   512, 6),
]


@pytest.mark.parametrize("lengths,Hq,Hkv,B,topk", CASES)
def test_varlen_equals_separate_calls(lengths, Hq, Hkv, B, topk):
    seqs, cu, (q, k, v) = packed(lengths, Hq, Hkv, B, topk, 900)
    out, lse = moba.fwd_varlen(q, k, v, cu, B, topk)
    torch.cuda.synchronize()
    assert moba.device_status() == moba.MOBA_OK
    for b, L in enumerate(lengths):
        if not L:
            continue
        a, e = int(cu[b]), int(cu[b + 1])
        o1, l1 = moba.fwd(q[a:e].contiguous(), k[a:e].contiguous(), v[a:e].contiguous(), B, topk)
        torch.cuda.synchronize()
        assert torch.equal(out[a:e], o1), b
        assert torch.equal(lse[:, a:e], l1), b


def test_varlen_against_the_oracle():
    lengths, Hq, Hkv, B, topk = [1500, 2100, 700], 4, 2, 256, 4
    seqs, cu, (q, k, v) = packed(lengths, Hq, Hkv, B, topk, 950)
    out, lse = moba.fwd_varlen(q, k, v, cu, B, topk)
    torch.cuda.synchronize()
    for b, (qs, ks, vs) in enumerate(seqs):
        a, e = int(cu[b]), int(cu[b + 1])
        kd = k[a:e].contiguous()
        kmean = moba.pool(kd, B)
        sel = moba.gate(q[a:e].contiguous(), kmean, Hkv, B, topk)
        torch.cuda.synchronize()
        full_check(qs, ks, vs, B, topk,
                   gpu=(out[a:e].cpu(), lse[:, a:e].cpu().numpy(), sel.cpu().numpy(), kmean.cpu().numpy()))


def test_varlen_graph_replay_follows_the_offsets():
    # the same buffers with new offsets must not replay the old batch's graph
    lengths, Hq, Hkv, B, topk = [2000, 3000], 4, 2, 256, 4
    seqs, cu, (q, k, v) = packed(lengths, Hq, Hkv, B, topk, 970)
    out = torch.empty_like(q)
    lse = torch.empty((Hq, q.shape[0]), dtype=torch.float32, device=q.device)
    first = None
    for _ in range(3):  # seen, captured, replayed
        moba.fwd_varlen(q, k, v, cu, B, topk, out=out, lse=lse)
        torch.cuda.synchronize()
        if first is None:
            first = (out.clone(), lse.clone())
        assert torch.equal(out, first[0]) and torch.equal(lse, first[1])
    cu2 = np.array([0, 2500, 5000], dtype=np.int64)
    for _ in range(3):
        moba.fwd_varlen(q, k, v, cu2, B, topk, out=out, lse=lse)
        torch.cuda.synchronize()
        for b in range(2):
            a, e = int(cu2[b]), int(cu2[b + 1])
            o1, l1 = moba.fwd(q[a:e].contiguous(), k[a:e].contiguous(), v[a:e].contiguous(), B, topk)
            torch.cuda.synchronize()
            assert torch.equal(out[a:e], o1) and torch.equal(lse[:, a:e], l1)
