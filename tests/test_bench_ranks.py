"""bench.py's multi-rank plumbing, as two gloo ranks on the CPU.

With --gpus N every rank runs its own sequence (weak scaling, no collective on
the data path); the only collective is a MAX all-reduce of the timings, and
the reference arm runs on rank 0 alone. These tests run that plumbing as two
processes on the gloo backend: the same calls the NCCL ranks make, minus the
GPU work.
"""
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime

    import bench
    import synth_inputs as si
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
        w = si.WORKLOADS["4k"]
        wr = bench.replica_workload(w, rank)
        # rank-dependent timings: rank 1 is slower in the first entry, rank 0 in the second
        mine = [10.0 + rank, 5.0 - rank, 1.5 * (rank + 1)]
        red = bench.max_over_ranks(mine, "cpu", world)
        # the reference arm: rank 0 only; the others return 0 without work
        ref_rc = None
        if rank != 0:
            class A:  # noqa: N801
                gpus, steps, warmup = world, 1, 3
            ref_rc = bench.run_reference(A, w)
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, wr.seed, wr.seqlen, red, ref_rc, bench.dist_env()))
    except Exception as e:  # noqa: BLE001
        q.put((rank, "error", repr(e)))


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        item = q.get(timeout=120)
        assert item[1] != "error", item
        res[item[0]] = item
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    seeds = {r: res[r][1] for r in res}
    assert seeds[0] != seeds[1], "each rank must draw its own sequence"
    assert res[0][2] == res[1][2], "same shape on every rank"
    for r in range(world):
        assert res[r][3] == [11.0, 5.0, 3.0], "MAX over ranks, element by element"
        assert res[r][5] == (r, world, r)
    assert res[1][4] == 0


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks x 4096 tokens x 10 steps over the slowest rank's 20 ms
    assert bench.job_tokens_per_s(2, 4096, 10, 20.0) == pytest.approx(2 * 4096 * 10 / 0.020)
    w = bench.si.WORKLOADS["128k"]
    assert bench.replica_workload(w, 0) == w
