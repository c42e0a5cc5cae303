"""The seeded input generator: known-answer and distribution checks (CPU)."""
import numpy as np
import torch

import synth_inputs as si


def test_splitmix64_reference_vector():
    # First outputs of SplitMix64 started at state 1234567, as published with
    # the generator's reference implementation (Vigna, splitmix64.c).
    L = si.lib()
    got = [L.synth_splitmix_output(1234567, i) for i in range(5)]
    assert got == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                   4593380528125082431, 16408922859458223821]


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(2000) * 3, rng.standard_normal(200) * 1e-3, [0.0, -0.0, 1.0, -2.5]])
    ours = si.f64_to_bf16_bits(x)
    # torch rounds fp32 -> bf16 nearest-even; go through fp32 only where that is exact
    x32 = x.astype(np.float32)
    exact = x32.astype(np.float64) == x
    ref = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours[exact], ref[exact])
    # ties-to-even at a bf16 half-way point: 1 + 2^-8 lies between 1 and 1 + 2^-7
    assert si.lib().synth_f64_to_bf16(1.0 + 2.0 ** -8) == 0x3F80
    assert si.lib().synth_f64_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82
    # just above half-way rounds up, which an fp32 detour would not see
    assert si.lib().synth_f64_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81


def test_normal_moments_and_counter_slices():
    w = si.Workload("t", 4096, 2, 1, 128, 512, 3, 7)
    q = np.empty((w.seqlen, w.heads_q, w.head_dim), dtype=np.uint16)
    si.fill_q(q.ctypes.data, w)
    x = si.bf16_bits_to_f64(q).ravel()
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    # any slice regenerates on its own (counter-based)
    part = np.empty((10, w.heads_q, w.head_dim), dtype=np.uint16)
    si.fill_q(part.ctypes.data, w, t0=1234, nrows=10, threads=1)
    assert np.array_equal(part, q[1234:1244])


def test_key_offsets_have_stated_norm_and_shift_blocks():
    w = si.Workload("t", 2048, 1, 2, 128, 256, 3, 11)
    mu = si.key_offsets(w)
    assert np.allclose(np.linalg.norm(mu, axis=-1), 0.5 * np.sqrt(128), rtol=1e-12)
    k = np.empty((w.seqlen, w.heads_kv, w.head_dim), dtype=np.uint16)
    si.fill_k(k.ctypes.data, w, mu)
    kf = si.bf16_bits_to_f64(k).reshape(w.nblocks, w.block_size, w.heads_kv, w.head_dim)
    blk_mean = kf.mean(axis=1).transpose(1, 0, 2)
    assert np.abs(blk_mean - mu).max() < 0.35  # N(0,1)/sqrt(256) noise, 128*8*2 draws


def test_upstream_gradient_stream_is_standard_normal_and_its_own():
    w = si.Workload("dout", 4096, 2, 1, 128, 512, 3, 5)
    do = si.bf16_bits_to_f64(si.make_dout(w, threads=2))
    q = si.bf16_bits_to_f64(si.make_qkv(w, threads=2)[0])
    assert abs(do.mean()) < 0.01 and abs(do.std() - 1.0) < 0.01
    assert not np.array_equal(do, q)
    part = np.empty((100, 2, 128), dtype=np.uint16)
    si.fill_dout(part.ctypes.data, w, t0=1000, nrows=100, threads=1)
    assert np.array_equal(si.bf16_bits_to_f64(part), do[1000:1100])
