"""bench.py's command line and host-side helpers, on the CPU (no GPU work)."""
import os
import subprocess
import sys

import numpy as np
import pytest

import synth_inputs as si

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("name,n", [("128k", 8), ("1m", 16), ("32k", 1), ("4k", 4096)])
def test_varlen_cuts_cover_the_workload_once(name, n):
    w = si.WORKLOADS[name]
    lengths, cu = bench.varlen_lengths(w, n)
    assert lengths.size == n and cu[0] == 0 and cu[-1] == w.seqlen
    assert np.all(lengths >= 1) and lengths.sum() == w.seqlen
    again, _ = bench.varlen_lengths(w, n)
    assert np.array_equal(lengths, again)  # seeded


def test_chunk_flops_of_the_whole_sequence_match_the_library_count():
    import block_sparse_long_fwd_b200 as moba
    for name in ("4k", "32k", "128k", "32k_dense"):
        w = si.WORKLOADS[name]
        want = moba.effective_flops(w.seqlen, w.heads_q, w.block_size, w.topk)
        assert bench.chunk_flops(w, 0) == pytest.approx(want, rel=1e-12)


@pytest.mark.parametrize("args", [
    ["--backward", "--chunk", "4"],
    ["--backward", "--varlen", "2"],
    ["--varlen", "3", "--chunk", "2"],
    ["--warmup", "2"],
    ["--cached-means"],
    ["--chunk", "-1"],
    ["--heads", "6:4"],
    ["--heads", "x"],
])
def test_incompatible_modes_are_rejected_before_any_gpu_work(args):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True, text=True,
                       timeout=300, cwd=ROOT)
    assert r.returncode == 2, r.stderr[-500:]
    assert "error" in r.stderr


@pytest.mark.parametrize("name,shape,flops", [
    ("4k", (4096, 1, 1, 512, 3), 2.28e9),
    ("32k", (32768, 1, 1, 2048, 3), 7.95e10),
    ("128k", (131072, 32, 8, 4096, 12), 8.30e13),
    ("1m", (1048576, 32, 8, 4096, 12), 7.91e14),
    ("10m", (10485760, 1, 1, 8192, 12), 5.04e14),
])
def test_workloads_and_their_flops_match_the_config_table(name, shape, flops):
    # the five configurations and their effective (selected-block) FLOPs:
    # 4*d*Hq per unmasked (query, key) pair, own block causal
    w = si.WORKLOADS[name]
    assert (w.seqlen, w.heads_q, w.heads_kv, w.block_size, w.topk) == shape and w.head_dim == 128
    assert bench.chunk_flops(w, 0) == pytest.approx(flops, rel=5e-3)
