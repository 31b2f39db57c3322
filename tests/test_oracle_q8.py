"""Pins of the 8-bit quantisers (CPU only).

* E4M3 rounding against a library routine (torch.float8_e4m3fn casts, which
  round to nearest even) on every value below the saturation point, plus the
  saturating closed form above it and a round trip through all 254 finite codes;
* int8 block quantisation against closed forms (absmax maps to +-127, zero
  block, ragged last block, block boundaries), and its codes (from a product
  with the block's fp32 reciprocal scale) against the textbook division by the
  scale: at most one step apart, on a 1e-4 fraction of elements at most;
* the diagnostic 8-bit simulation reduces to the dequantised V for S = 1 and
  stays within the quantisation error budget of the exact oracle;
* the simulation's folded form (each block's V scale carried inside P) against
  the recipe written out block by block (each block's 8-bit product dequantised
  by its own scale and accumulated across blocks): equal to rounding wherever no
  P code is subnormal, with a ragged last block and block-scale ratios down to
  2^-5; both reduce to the mean of the dequantised V when every score is equal;
  planted mistakes in the fold (another block's scale, an exponent off by one)
  break the equality.
"""
import numpy as np
import pytest
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


def _v_with_scaled_blocks(rng, S, H, D, factors):
    """N(0,1) values with the 64-token block t multiplied by factors[t] (powers of two: exact)."""
    v = rng.standard_normal((1, S, H, D)).astype(np.float32)
    for t, f in enumerate(factors):
        v[:, 64 * t:64 * (t + 1)] *= np.float32(f)
    return v


def _blockwise_case():
    rng = np.random.default_rng(11)
    S, H, D = 200, 2, 128                           # blocks of 64, 64, 64 and a ragged 8
    q = (rng.standard_normal((1, S, H, D)) * 0.5).astype(np.float32)
    k = (rng.standard_normal((1, S, H, D)) * 0.5).astype(np.float32)
    v = _v_with_scaled_blocks(rng, S, H, D, [1.0, 2.0 ** -3, 2.0 ** -5, 0.5])
    return q, k, v


def test_q8_folded_form_equals_blockwise_accumulation():
    q, k, v = _blockwise_case()
    S = q.shape[1]
    _, _, sv = q8.quant_e4m3(v)
    ratios = sv / sv.max(axis=2, keepdims=True)
    assert ratios.min() <= 2.0 ** -5 and len(np.unique(ratios)) >= 4      # the fold really shifts exponents
    # no P code is subnormal: the smallest weight p = exp(s - m) times 448 * ratio stays >= 2^-6
    for h in range(q.shape[2]):
        p = oracle.softmax_matrix(q, k, 0, h)
        pmin = (p / p.max(axis=1, keepdims=True)).min()
        assert 448.0 * pmin * 0.9 * ratios[0, h].min() >= 2.0 ** -6
    o_f, l_f = q8.attn_fwd_q8_sim(q, k, v)
    o_b, l_b = q8.attn_fwd_q8_blockwise(q, k, v)
    np.testing.assert_allclose(o_f, o_b, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l_f, l_b, rtol=0, atol=1e-12)
    rows = np.array([0, 63, 64, 199])
    o_r, _ = q8.attn_fwd_q8_blockwise(q, k, v, rows=rows, heads=[1])
    np.testing.assert_allclose(o_r[:, :, 0], o_b[:, rows, 1], rtol=1e-12, atol=1e-13)
    assert S == 200


def test_q8_uniform_scores_reduce_to_mean_of_dequantised_v():
    rng = np.random.default_rng(12)
    S, H, D = 150, 2, 16
    q = np.zeros((1, S, H, D), dtype=np.float32)
    k = rng.standard_normal((1, S, H, D)).astype(np.float32)
    v = _v_with_scaled_blocks(rng, S, H, D, [1.0, 0.25, 4.0])
    _, vals, sv = q8.quant_e4m3(v)
    deq = vals * np.repeat(sv, 64, axis=2)[:, :, :S].transpose(0, 2, 1)[:, :, :, None]
    want = np.broadcast_to(deq.mean(axis=1, keepdims=True), (1, S, H, D))
    for fn in (q8.attn_fwd_q8_sim, q8.attn_fwd_q8_blockwise):
        o, lse = fn(q, k, v)
        np.testing.assert_allclose(o, want, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lse, np.log(S), rtol=0, atol=1e-12)


def test_q8_forms_differ_only_by_subnormal_codes_on_peaky_scores():
    rng = np.random.default_rng(13)
    S, H, D = 256, 1, 128
    q = (rng.standard_normal((1, S, H, D)) * 3).astype(np.float32)   # weights far below 2^-6 / 448
    k = rng.standard_normal((1, S, H, D)).astype(np.float32)
    v = _v_with_scaled_blocks(rng, S, H, D, [1.0, 2.0 ** -4, 1.0, 2.0 ** -2])
    o_f, _ = q8.attn_fwd_q8_sim(q, k, v)
    o_b, _ = q8.attn_fwd_q8_blockwise(q, k, v)
    rel = np.linalg.norm(o_f - o_b) / np.linalg.norm(o_b)
    assert 0 < rel < 1e-2, rel        # subnormal P codes round on different grids; nothing else differs


@pytest.mark.parametrize("kind", ["neighbour_block_scale", "exponent_off_by_one", "unfolded_scale"])
def test_q8_planted_fold_mistakes_are_caught(monkeypatch, kind):
    good = q8._fold_factor

    def bad(sv_bh, S, block):
        f = good(sv_bh, S, block)
        if kind == "neighbour_block_scale":        # key j takes the scale of the block before its own
            return np.concatenate([f[:block], f[:-block]])
        if kind == "exponent_off_by_one":          # 2^(k - kmax + 1) instead of 2^(k - kmax)
            return np.minimum(2.0 * f, 1.0)
        return np.ones_like(f)                     # the block scale forgotten
    monkeypatch.setattr(q8, "_fold_factor", bad)
    q, k, v = _blockwise_case()
    o_f, _ = q8.attn_fwd_q8_sim(q, k, v)
    o_b, _ = q8.attn_fwd_q8_blockwise(q, k, v)
    assert np.linalg.norm(o_f - o_b) / np.linalg.norm(o_b) > 1e-3


def test_int8_codes_by_reciprocal_product_match_division_but_for_rare_ties():
    # The quantiser forms its codes as rint(fp32(x * fp32(127 / absmax))); the textbook form is
    # rint(x / (absmax / 127)).  Both round the same real quotient up to an fp32 rounding or two,
    # so codes differ by at most one step and only where the quotient sits within an ulp of a
    # half-integer: the reading of the pages' "absmax/127 scale" does not change the recipe.
    rng = np.random.default_rng(21)
    x = rng.standard_normal((1, 4096, 4, 128)).astype(np.float32)
    codes, scale = q8.quant_int8(x)
    amax = q8.block_absmax(x)
    per = np.repeat(amax, 64, axis=2)[:, :, :4096].transpose(0, 2, 1)[:, :, :, None].astype(np.float64)
    textbook = np.clip(np.rint(x.astype(np.float64) / (per / 127.0)), -127, 127)
    diff = np.abs(codes.astype(np.int64) - textbook.astype(np.int64))
    assert diff.max() <= 1
    assert np.count_nonzero(diff) <= 1e-4 * diff.size
