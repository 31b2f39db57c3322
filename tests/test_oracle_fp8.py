"""Pins of the FP8 GEMM oracle (oracle/fp8_gemm.py) to things other than itself (CPU only).

The e4m3 rounding itself is pinned in test_oracle_q8.py (torch's float8_e4m3fn cast,
every code's round trip).  Here:
* exact inputs: rows that are a power-of-two scale times e4m3 grid values with
  absmax 448 x scale quantise without error, so the recipe reduces to the plain
  fp64 product X W^T (a library matmul);
* the e4m3 error bound: every dequantised element is within half a code step of
  the input (2^-4 relative for normal codes, 2^-10 x scale below 2^-6);
* invariants: the largest code of every nonzero row (and of W) is +-448; zero rows
  give zero codes, scale 1 and zero output; scaling a row by a power of two scales
  its scale only;
* shapes: Y is [M, N] for X [M, K] and W [N, K] (a transposed operand fails);
* the recipe's error against the unquantised product is the e4m3 level (a few %).
"""
import numpy as np
import pytest

from oracle import fp8_gemm as fg
from oracle.quant8 import e4m3_round


def grid_values(rng, shape):
    """Random e4m3-representable magnitudes with random signs (fp64)."""
    raw = rng.standard_normal(shape) * 100
    return e4m3_round(raw)


def test_exact_inputs_reduce_to_the_plain_product():
    rng = np.random.default_rng(0)
    M, N, K = 7, 5, 64
    x = grid_values(rng, (M, K))
    x[:, 0] = 448.0                               # absmax of every row is 448
    x *= (2.0 ** rng.integers(-6, 4, size=(M, 1)))  # power-of-two row scales
    w = grid_values(rng, (N, K))
    w[0, 0] = -448.0
    w *= 2.0 ** -3
    bits, xv, sx = fg.quant_rows(x.astype(np.float32))
    np.testing.assert_array_equal(xv * sx[:, None].astype(np.float64), x)
    _, wv, sw = fg.quant_tensor(w.astype(np.float32))
    np.testing.assert_array_equal(wv * float(sw), w)
    np.testing.assert_allclose(fg.fp8_linear(x.astype(np.float32), w.astype(np.float32)), x @ w.T,
                               rtol=1e-14, atol=0)


def test_dequantisation_error_within_half_a_code_step():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((40, 300)) * np.exp(rng.standard_normal((40, 1)) * 3)).astype(np.float32)
    _, xv, sx = fg.quant_rows(x)
    deq = xv * sx[:, None].astype(np.float64)
    xf = x.astype(np.float64)
    mag = np.abs(xf) / sx[:, None]                 # in code units
    bound = np.where(mag >= 2.0 ** -6, 2.0 ** -4 * mag, 2.0 ** -10) * sx[:, None] * (1 + 1e-6)
    assert np.all(np.abs(deq - xf) <= bound)


def test_largest_code_is_448_and_zero_rows():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((9, 33)).astype(np.float32)
    x[4] = 0.0
    bits, xv, sx = fg.quant_rows(x)
    big = np.abs(xv).max(axis=1)
    assert np.all(big[np.arange(9) != 4] == 448.0)
    assert np.all(bits[4] == 0) and sx[4] == 1.0
    w = rng.standard_normal((6, 33)).astype(np.float32)
    _, wv, sw = fg.quant_tensor(w)
    assert np.abs(wv).max() == 448.0
    y = fg.fp8_linear(x, w)
    assert y.shape == (9, 6) and np.all(y[4] == 0.0)


def test_power_of_two_row_scaling_moves_only_the_scale():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((3, 50)).astype(np.float32)
    b1, v1, s1 = fg.quant_rows(x)
    b2, v2, s2 = fg.quant_rows(x * np.float32(8.0))
    np.testing.assert_array_equal(b1, b2)
    np.testing.assert_array_equal(s2, s1 * np.float32(8.0))


def test_operand_orientation():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((4, 16)).astype(np.float32)
    w = rng.standard_normal((3, 16)).astype(np.float32)
    assert fg.fp8_linear(x, w).shape == (4, 3)
    with pytest.raises(ValueError):
        fg.fp8_linear(x, w.T.copy())


def test_recipe_error_against_the_unquantised_product():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((64, 512)).astype(np.float32)
    w = (rng.standard_normal((96, 512)) * 0.02).astype(np.float32)
    exact = x.astype(np.float64) @ w.astype(np.float64).T
    y = fg.fp8_linear(x, w)
    rel = np.linalg.norm(y - exact) / np.linalg.norm(exact)
    assert 5e-3 < rel < 8e-2, rel          # e4m3's 3 mantissa bits on both operands
