"""The seeded input generator and the workload shapes (CPU only)."""
import os

import numpy as np
import pytest

import synth
from conftest import read_golden


def test_c_generator_matches_numpy_twin():
    for seed, stream, first in [(0, 0, 0), (0, 1, 12345), (7, 3, 10 ** 9)]:
        n = 20000
        c_f64 = synth.normal_f64(seed, stream, n, first)
        np_f64 = synth.normal_f64_np(seed, stream, n, first)
        np.testing.assert_allclose(c_f64, np_f64, rtol=1e-13, atol=1e-13)
        c_bits = synth.normal_bf16(seed, stream, n, first)
        np_bits = synth.f64_to_bf16_bits(np_f64)
        # libm vs numpy transcendental ulps may flip a bf16 rounding very rarely
        assert np.count_nonzero(c_bits != np_bits) <= 2


def test_bf16_rounding_is_nearest_even():
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> even (1.0); 1 + 3*2^-8 -> 1 + 2^-6
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0])
    bits = synth.f64_to_bf16_bits(x)
    back = synth.bf16_bits_to_f32(bits).astype(np.float64)
    np.testing.assert_array_equal(back, [1.0, 1.0, 1.0 + 2 ** -6, -2.5, 0.0])


def test_ranges_are_counter_based():
    whole = synth.normal_bf16(0, 2, 5000)
    part = synth.normal_bf16(0, 2, 1000, first=3000)
    np.testing.assert_array_equal(whole[3000:4000], part)
    assert not np.array_equal(synth.normal_bf16(0, 1, 1000), synth.normal_bf16(0, 2, 1000))
    assert not np.array_equal(synth.normal_bf16(0, 1, 1000), synth.normal_bf16(1, 1, 1000))


def test_moments_are_standard_normal():
    z = synth.normal_f64(0, 0, 2_000_000)
    assert abs(z.mean()) < 3e-3
    assert abs(z.var() - 1.0) < 5e-3
    assert abs(np.mean(z ** 3)) < 1e-2            # symmetric
    assert abs(np.mean(z ** 4) - 3.0) < 3e-2      # normal kurtosis


def test_token_counts_golden(golden_dir):
    for frames, h, w, tokens in read_golden(os.path.join(golden_dir, "token_counts.txt")):
        assert synth.tokens_for_video(int(frames), int(h), int(w)) == int(tokens)
    with pytest.raises(ValueError):
        synth.tokens_for_video(80, 720, 1280)


def test_cost_model_golden(golden_dir):
    for name, B, S, H, D, flop in read_golden(os.path.join(golden_dir, "cost_model.txt")):
        w = synth.WORKLOADS[name]
        assert (w.B, w.S, w.H, w.D) == (int(B), int(S), int(H), int(D))
        assert w.fwd_flop == float(flop)


def test_sample_rows():
    r = synth.sample_rows(75600, 256)
    assert len(r) == 256 and len(set(r.tolist())) == 256
    assert r[0] == 0 and r[-1] == 75599 and np.all(np.diff(r) > 0)
    np.testing.assert_array_equal(r, synth.sample_rows(75600, 256))
    k = synth.sample_rows(75600, 256, stream=synth.STREAM_KROWS)
    assert not np.array_equal(r, k)
    np.testing.assert_array_equal(synth.sample_rows(100, 256), np.arange(100))


def test_peaky_heads_and_scaling():
    w = synth.WORKLOADS["wan1.3b_480p_cfg"]
    heads = synth.peaky_heads(w.H, w.peaky_frac)
    assert len(heads) == 1 and 0 <= heads[0] < 12
    assert synth.peaky_heads(40, 0.1) == synth.peaky_heads(40, 0.1) and len(synth.peaky_heads(40, 0.1)) == 4
    x = synth.make_inputs(w, S=64)
    plain = synth.make_tensor((2, 64, 12, 128), 0, synth.STREAM_Q)
    fq = synth.bf16_bits_to_f32(x["q"])
    fp = synth.bf16_bits_to_f32(plain)
    for h in range(12):
        want = fp[:, :, h] * (2.0 if h in heads else 1.0)
        np.testing.assert_array_equal(fq[:, :, h], want)
