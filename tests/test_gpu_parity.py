"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Small cases check every row; the large workloads (128K, 1M, 10M tokens) run
in the configuration the benchmark times and are checked on sampled rows
(edge rows plus a seeded uniform sample), which the oracle computes one by
one. Tolerances live in parity_helpers.
"""
import os

import numpy as np
import pytest

import oracle
import synth_inputs as si
from parity_helpers import full_check, make_inputs, run_gpu

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)


SMALL = [
    # S,    Hq, Hkv, B,   topk, seed
    (1,     1,  1,   128, 3,    1),     # one token
    (100,   2,  1,   128, 3,    2),     # shorter than a block
    (1000,  4,  2,   128, 3,    3),     # ragged tail, GQA
    (1536,  3,  1,   128, 4,    4),     # group size 3
    (2048,  8,  8,   256, 2,    5),     # MHA
    (4096,  2,  1,   128, 1,    6),     # topk 1: own block only
    (1536,  2,  1,   128, 20,   7),     # topk >= blocks: full causal attention
    (2125,  2,  1,   256, 5,    8),     # ragged, several routed blocks
    (8192,  4,  1,   512, 9,    9),     # many past blocks per row
    (3000,  1,  1,   256, 4,    10),    # one head per group: own tiles paired by token, ragged last pair
    (2900,  2,  2,   512, 3,    11),    # paired own tiles, last pair without its second tile
    (4096,  1,  1,   512, 8,    12),    # topk >= blocks, one head: the dense path, paired own tiles
    (3000,  4,  2,   256, 64,   13),    # dense path, GQA, ragged
    (8192,  2,  1,   128, 20,   14),    # 19 past blocks kept per row (24-entry top-k lists)
    (12000, 2,  1,   128, 40,   15),    # 39 past blocks kept per row (48-entry lists), ragged
]


@pytest.mark.parametrize("S,Hq,Hkv,B,topk,seed", SMALL)
def test_small_all_rows(S, Hq, Hkv, B, topk, seed):
    w, q, k, v = make_inputs(S, Hq, Hkv, B, topk, seed)
    stats = full_check(q, k, v, B, topk)
    print(stats)


@pytest.mark.parametrize("window,heads", [(128, (4, 2)), (384, (4, 2)), (1024, (4, 2)), (384, (2, 2)), (640, (1, 1))])
def test_query_windows(monkeypatch, window, heads):
    # (1, 1) and (2, 2): one head per group, windows rounded to 256 tokens for paired own tiles
    S, (Hq, Hkv), B, topk = 2125, heads, 256, 4
    w, q, k, v = make_inputs(S, Hq, Hkv, B, topk, 40 + window + Hq)
    monkeypatch.setenv("MOBA_WINDOW", str(window))
    stats = full_check(q, k, v, B, topk)
    print(window, stats)


@pytest.mark.parametrize("name", ["4k", "32k"])
def test_workload_all_rows(name):
    w = si.WORKLOADS[name]
    q, k, v = si.make_qkv(w)
    stats = full_check(q, k, v, w.block_size, w.topk)
    print(name, stats)


def test_deterministic_bits():
    w = si.WORKLOADS["32k"]
    q, k, v = si.make_qkv(w)
    a = run_gpu(q, k, v, w.block_size, w.topk)
    b = run_gpu(q, k, v, w.block_size, w.topk)
    assert torch.equal(a[0], b[0])
    for x, y in zip(a[1:], b[1:]):
        assert np.array_equal(x, y)


def sample_rows(w, n, seed):
    rng = np.random.default_rng(seed)
    S, Hq, B = w.seqlen, w.heads_q, w.block_size
    t = rng.choice(S, size=n, replace=False).astype(np.int64)
    edge = np.array([0, B - 1, B, 2 * B - 1, S - 1, S // 2], dtype=np.int64)
    t = np.concatenate([edge, t])
    h = rng.integers(0, Hq, size=t.size).astype(np.int32)
    return t, h


@pytest.mark.parametrize("name,nrows", [("32k_dense", 512), ("128k_dense", 128), ("128k_b512", 256)])
def test_dense_workload_sampled_rows(name, nrows):
    # topk >= number of blocks is full causal attention; the library runs it
    # as one causal pass (no gate scores, no routing) and must match the
    # oracle. 128k_b512: finer blocks (512 tokens, top-48) through the same path
    w = si.WORKLOADS[name]
    q, k, v = si.make_qkv(w)
    rows = sample_rows(w, nrows, w.seed + 2000)
    stats = full_check(q, k, v, w.block_size, w.topk, rows=rows)
    print(name, stats)


def test_dense_path_launches_no_router():
    import block_sparse_long_fwd_b200 as moba
    S, Hq, Hkv, B, topk = 8192, 2, 2, 512, 16
    from parity_helpers import to_dev
    w, q, k, v = make_inputs(S, Hq, Hkv, B, topk, 21)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    moba.profile_begin()
    moba.fwd(qd, kd, vd, B, topk)
    _, launches, calls = moba.profile_end()
    torch.cuda.synchronize()
    # one window: selection fill, unit list, attention, merge
    assert calls == 1 and launches == 4, launches


def _bf16_bits(x):
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def test_rescale_decided_per_row():
    # Rows of one warp that move their softmax reference at different steps:
    # in the second 128-key step, even rows see logits ~10 nats above the
    # first step's (a reference move) and odd rows ~10 nats below (none).
    # The O rescale is per row but its TMEM accesses are warp-collective.
    S, B = 512, 512
    rng = np.random.default_rng(5)
    q = rng.normal(0, 0.1, (S, 1, 128)).astype(np.float32)
    k = rng.normal(0, 0.1, (S, 1, 128)).astype(np.float32)
    v = rng.normal(0, 1.0, (S, 1, 128)).astype(np.float32)
    sign = np.where(np.arange(S) % 2 == 0, 1.0, -1.0)
    q[:, 0, 0] = 10.6 * sign
    k[128:, 0, 0] = 10.6
    stats = full_check(_bf16_bits(q), _bf16_bits(k), _bf16_bits(v), B, 1)
    print(stats)


def test_bounded_wait_reports_timeout():
    import block_sparse_long_fwd_b200 as moba
    assert moba.selftest_bounded_wait(20000) == moba.MOBA_ERR_DEVICE_TIMEOUT
    assert moba.device_status() == 0  # cleared by the read


def test_an_earlier_device_error_is_reported_by_the_next_call():
    # a kernel whose bounded wait runs out, launched without reading the
    # status: the next call returns that code before launching, once
    import block_sparse_long_fwd_b200 as moba
    S, Hq, Hkv, B, topk = 1000, 2, 1, 256, 3
    _, q, k, v = make_inputs(S, Hq, Hkv, B, topk, 5)
    qd, kd, vd = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda() for a in (q, k, v))
    stream = torch.cuda.current_stream().cuda_stream
    assert moba.lib().moba_selftest_bounded_wait_async(20000, stream) == moba.MOBA_OK
    torch.cuda.synchronize()
    with pytest.raises(moba.MobaError) as err:
        moba.fwd(qd, kd, vd, B, topk)
    assert err.value.code == moba.MOBA_ERR_DEVICE_TIMEOUT
    out, lse = moba.fwd(qd, kd, vd, B, topk)  # reported once: this call runs
    torch.cuda.synchronize()
    assert moba.device_status() == moba.MOBA_OK
    assert torch.isfinite(lse).all()


def test_sync_mode_returns_the_device_status_from_the_call(monkeypatch):
    import block_sparse_long_fwd_b200 as moba
    monkeypatch.setenv("MOBA_SYNC", "1")
    stream = torch.cuda.current_stream().cuda_stream
    assert moba.lib().moba_selftest_bounded_wait_async(20000, stream) == moba.MOBA_ERR_DEVICE_TIMEOUT
    S, Hq, Hkv, B, topk = 1000, 2, 1, 256, 3
    _, q, k, v = make_inputs(S, Hq, Hkv, B, topk, 6)
    qd, kd, vd = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda() for a in (q, k, v))
    moba.fwd(qd, kd, vd, B, topk)  # a clean call returns MOBA_OK after synchronising
    assert moba.device_status() == moba.MOBA_OK


def test_device_check_is_recorded_and_the_access_skipped():
    # the merge kernel on router tables that point outside the list: it must
    # record the check failure instead of reading there
    import block_sparse_long_fwd_b200 as moba
    stream = torch.cuda.current_stream().cuda_stream
    assert moba.lib().moba_selftest_device_check(stream) == moba.MOBA_ERR_DEVICE_CHECK
    assert moba.device_status() == moba.MOBA_OK  # read and cleared
    # the library still works afterwards
    S, Hq, Hkv, B, topk = 1000, 2, 1, 256, 3
    _, q, k, v = make_inputs(S, Hq, Hkv, B, topk, 8)
    stats = full_check(q, k, v, B, topk)
    print(stats)


def test_failed_scratch_allocation_returns_oom(monkeypatch):
    # the test hook adds 2^50 bytes to the scratch request, so the
    # stream-ordered allocation fails for real and the call reports it
    import block_sparse_long_fwd_b200 as moba
    from parity_helpers import to_dev
    S, Hq, Hkv, B, topk = 2000, 2, 1, 256, 3
    _, q, k, v = make_inputs(S, Hq, Hkv, B, topk, 9)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    monkeypatch.setenv("MOBA_TEST_SCRATCH_PAD", str(1 << 50))
    with pytest.raises(moba.MobaError) as err:
        moba.fwd(qd, kd, vd, B, topk)
    assert err.value.code == moba.MOBA_ERR_OOM
    assert "scratch allocation" in str(err.value)
    monkeypatch.delenv("MOBA_TEST_SCRATCH_PAD")
    torch.cuda.synchronize()
    assert moba.device_status() == moba.MOBA_OK
    out, lse = moba.fwd(qd, kd, vd, B, topk)  # and the next call runs
    torch.cuda.synchronize()
    assert torch.isfinite(lse).all() and moba.device_status() == moba.MOBA_OK


def test_host_entry_point_matches_device_entry_point():
    import block_sparse_long_fwd_b200 as moba
    S, Hq, Hkv, B, topk = 3000, 4, 2, 256, 3
    w, q, k, v = make_inputs(S, Hq, Hkv, B, topk, 77)
    to_t = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    out_h, lse_h = moba.fwd_host(to_t(q).pin_memory(), to_t(k).pin_memory(), to_t(v).pin_memory(), B, topk)
    out_d, lse_d, _, _ = run_gpu(q, k, v, B, topk)
    assert torch.equal(out_h, out_d)
    assert np.array_equal(lse_h.numpy(), lse_d)


@pytest.mark.parametrize("S,Hq,Hkv,B,topk,window,pinned", [
    (3000, 4, 2, 256, 3, 256, True),    # 12 windows, one per block
    (3000, 6, 2, 256, 5, 384, True),    # G = 3 (Q gathered by cp.async); windows straddle blocks
    (3000, 4, 2, 256, 3, 384, False),   # pageable host buffers
    (1000, 2, 1, 256, 8, 256, True),    # topk >= blocks: no gate, windows still pipelined
])
def test_host_entry_point_pipelined_over_windows(monkeypatch, S, Hq, Hkv, B, topk, window, pinned):
    # moba_fwd_host copies each window's rows up ahead of its kernels and its
    # outputs back behind them; results are those of the device entry point
    import block_sparse_long_fwd_b200 as moba
    w, q, k, v = make_inputs(S, Hq, Hkv, B, topk, 91)
    to_t = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    host = [to_t(x) for x in (q, k, v)]
    if pinned:
        host = [x.pin_memory() for x in host]
    monkeypatch.setenv("MOBA_WINDOW", str(window))  # the same windows on both paths
    out_h, lse_h = moba.fwd_host(*host, B, topk)
    out_h2, lse_h2 = moba.fwd_host(*host, B, topk)
    out_d, lse_d, _, _ = run_gpu(q, k, v, B, topk)
    assert torch.equal(out_h, out_d) and torch.equal(out_h2, out_d)
    assert np.array_equal(lse_h.numpy(), lse_d) and np.array_equal(lse_h2.numpy(), lse_d)
    assert moba.device_status() == moba.MOBA_OK


def test_repeated_calls_replay_a_graph_with_identical_results():
    # the third call with the same buffers replays a captured CUDA graph
    import block_sparse_long_fwd_b200 as moba
    from parity_helpers import to_dev
    w = si.WORKLOADS["4k"]
    q, k, v = si.make_qkv(w)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    out = torch.empty_like(qd)
    lse = torch.empty((w.heads_q, w.seqlen), dtype=torch.float32, device="cuda")
    moba.fwd(qd, kd, vd, w.block_size, w.topk, out=out, lse=lse)
    first = (out.clone(), lse.clone())
    for _ in range(3):
        out.zero_()
        lse.zero_()
        moba.fwd(qd, kd, vd, w.block_size, w.topk, out=out, lse=lse)
        torch.cuda.synchronize()
        assert torch.equal(out, first[0]) and torch.equal(lse, first[1])
    assert moba.device_status() == 0
