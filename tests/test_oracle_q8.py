"""Pins of the 8-bit quantisers (CPU only).

* E4M3 rounding against a library routine (torch.float8_e4m3fn casts, which
  round to nearest even) on every value below the saturation point, plus the
  saturating closed form above it and a round trip through all 254 finite codes;
* int8 block quantisation against closed forms (absmax maps to +-127, zero
  block, ragged last block, block boundaries);
* the diagnostic 8-bit simulation reduces to the dequantised V for S = 1 and
  stays within the quantisation error budget of the exact oracle.
"""
import numpy as np
import torch

import oracle
from oracle import quant8 as q8


def test_e4m3_round_matches_torch_cast():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * 50,
        rng.uniform(-463.9, 463.9, 100000).astype(np.float32),
        (rng.standard_normal(50000) * 1e-2).astype(np.float32),
        np.float32(2.0) ** np.arange(-12, 9, dtype=np.float32),
        np.array([0.0, -0.0, 2 ** -10, 3 * 2 ** -10, 2 ** -9 * 1.5, 447.9, 448.0, 463.9], dtype=np.float32),
    ])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn)
    np.testing.assert_array_equal(q8.e4m3_round(x), ref.float().numpy().astype(np.float64))
    np.testing.assert_array_equal(q8.e4m3_bits(x), ref.view(torch.uint8).numpy())


def test_e4m3_saturates_and_round_trips_all_codes():
    np.testing.assert_array_equal(q8.e4m3_round(np.array([464.0, 500.0, 1e6, -1e9])),
                                  [448.0, 448.0, 448.0, -448.0])
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    np.testing.assert_array_equal(q8.e4m3_bits(vals)[codes != 0x80], codes[codes != 0x80])
    np.testing.assert_array_equal(q8.e4m3_round(vals), vals.astype(np.float64))


def test_int8_block_quantisation_closed_forms():
    B, S, H, D = 1, 130, 2, 4          # blocks of 64, 64, 2 tokens
    x = np.zeros((B, S, H, D), dtype=np.float32)
    x[0, 10, 0, 1] = -5.0               # block 0 head 0: absmax 5
    x[0, 20, 0, 2] = 2.5
    x[0, 70, 0, 0] = 3.0                # block 1 head 0: absmax 3
    x[0, 129, 1, 3] = 0.75              # block 2 head 1 (ragged, 2 tokens)
    codes, scale = q8.quant_int8(x)
    assert scale.shape == (1, 2, 3)
    np.testing.assert_array_equal(scale[0, 0], np.float32([5.0 / 127, 3.0 / 127, 1.0]))
    np.testing.assert_array_equal(scale[0, 1], np.float32([1.0, 1.0, 0.75 / 127]))
    assert codes[0, 10, 0, 1] == -127 and codes[0, 70, 0, 0] == 127 and codes[0, 129, 1, 3] == 127
    assert codes[0, 20, 0, 2] == 64     # 2.5 / (5/127) = 63.5 -> ties to even 64
    assert np.count_nonzero(codes) == 4


def test_int8_codes_dequantise_within_half_step():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((1, 200, 3, 128)).astype(np.float32)
    codes, scale = q8.quant_int8(x)
    per = np.repeat(scale, 64, axis=2)[:, :, :200].transpose(0, 2, 1)[:, :, :, None]
    err = np.abs(codes * per.astype(np.float64) - x)
    assert np.all(err <= per * 0.5 * (1 + 1e-6))
    assert np.abs(codes).max() == 127


def test_e4m3_block_quantisation():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((1, 100, 2, 16)).astype(np.float32)
    bits, vals, scale = q8.quant_e4m3(x)
    amax = np.abs(x[:, :64]).max(axis=(1, 3))
    # power-of-two scales: 2^k with 2^(k-1) < absmax/448 <= 2^k
    s0 = scale[:, :, 0].astype(np.float64)
    assert np.all(np.log2(s0) == np.round(np.log2(s0)))
    assert np.all(s0 >= amax / 448.0) and np.all(s0 / 2 < amax / 448.0)
    np.testing.assert_array_equal(q8.pow2_ceil_f32(np.float32([0.25, 0.3, 1.0, 3e-41, 5.0])),
                                  np.float32([0.25, 0.5, 1.0, 2.0 ** -134, 8.0]))
    deq = vals * np.repeat(scale, 64, axis=2)[:, :, :100].transpose(0, 2, 1)[:, :, :, None]
    rel = np.abs(deq - x) / np.maximum(np.abs(x), 1e-3)
    assert np.percentile(rel, 99) < 0.07


def test_q8_sim_single_key_and_error_budget():
    rng = np.random.default_rng(3)
    v = rng.standard_normal((1, 1, 2, 16)).astype(np.float32)
    q = rng.standard_normal((1, 1, 2, 16)).astype(np.float32)
    o, _ = q8.attn_fwd_q8_sim(q, q, v)
    _, vals, scale = q8.quant_e4m3(v)
    np.testing.assert_allclose(o[0, 0], vals[0, 0] * scale[0, :, 0][:, None], rtol=1e-12)
    x = {n: rng.standard_normal((1, 256, 2, 128)).astype(np.float32) for n in "qkv"}
    oe, le = oracle.attn_fwd(x["q"], x["k"], x["v"])
    os_, ls = q8.attn_fwd_q8_sim(x["q"], x["k"], x["v"])
    rel = np.linalg.norm(os_ - oe) / np.linalg.norm(oe)
    assert 0.01 < rel < 0.045, rel
    assert np.abs(ls - le).max() < 0.05
