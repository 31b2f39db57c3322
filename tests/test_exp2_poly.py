"""The polynomial 2^x the kernels use for part of their exponentials (CPU).

The kernel's steps are emulated in numpy fp32 (round-to-integer by adding
1.5 * 2^23, the same Horner chain, exponent-field add) and checked against
the exact 2^x: relative error <= 1e-4 over the softmax's whole input range,
a tenth of bf16's rounding step.  The degree-2 pair form of the 8-bit forward,
whose results are rounded to e4m3, is held to 1.8e-3, under a thirtieth of
e4m3's half step.  The coefficients are read from the CUDA header, so a change
there is caught here; they are those the fitting script produces.
"""
import os
import re

import numpy as np

from conftest import ROOT

HEADER = os.path.join(ROOT, "video_dit_full_b200", "csrc", "sm100_ptx.cuh")


def header_coefficients():
    body = open(HEADER).read()
    body = body[body.index("float exp2_poly3"):]
    body = body[:body.index("\n}")]
    # fmaf(c3, f, c2); fmaf(p, f, c1); fmaf(p, f, c0): the only literals with digits after the point
    c3, c2, c1, c0 = [float(x) for x in re.findall(r"(-?\d+\.\d+)f", body)]
    return c0, c1, c2, c3


def emulate(x):
    f32 = np.float32
    c0, c1, c2, c3 = (f32(c) for c in header_coefficients())
    x = np.maximum(x.astype(f32), f32(-125.0))
    j = (x + f32(12582912.0)).astype(f32)
    f = (x - (j - f32(12582912.0))).astype(f32)
    fma = lambda a, b, c: (a.astype(np.float64) * b + c).astype(f32)   # one rounding, like FFMA
    p = fma(np.full_like(f, c3), f, c2)
    p = fma(p, f, c1)
    p = fma(p, f, c0)
    bits = p.view(np.int32) + (j.view(np.int32) << 23)
    return bits.view(f32).astype(np.float64)


def test_relative_error_over_softmax_range():
    x = np.concatenate([np.linspace(-125, 9, 400001), np.random.default_rng(0).uniform(-30, 9, 200000)])
    x32 = x.astype(np.float32).astype(np.float64)
    rel = np.abs(emulate(x32) / np.exp2(x32) - 1)
    assert rel.max() <= 1e-4, rel.max()


def test_clamp_keeps_results_normal_and_tiny():
    y = emulate(np.array([-np.inf, -1000.0, -125.0], dtype=np.float64))
    assert np.all(y > 0) and np.all(y < 2.0 ** -124) and np.all(y >= np.finfo(np.float32).tiny)


def test_coefficients_are_the_fitted_ones():
    from video_dit_full_b200.fit_exp2_poly import fit
    c = fit(3)
    np.testing.assert_allclose(header_coefficients(), c, rtol=1e-6)


# ---- the degree-2 pair form the 8-bit forward uses (its results are rounded to e4m3 next) ----

def header_coefficients_deg2():
    body = open(HEADER).read()
    body = body[body.index("float2 exp2_poly2_x2"):]
    body = body[:body.index("\n}")]
    # ffma2(c2, f, c1) then ffma2(p, f, c0), each constant written twice (both halves of the pair)
    vals = [float(x) for x in re.findall(r"(-?\d+\.\d{3,})f", body)]
    c2, c1, c0 = vals[0], vals[2], vals[4]
    assert vals[1] == c2 and vals[3] == c1 and vals[5] == c0
    return c0, c1, c2


def emulate_deg2(x):
    f32 = np.float32
    c0, c1, c2 = (f32(c) for c in header_coefficients_deg2())
    x = np.maximum(x.astype(f32), f32(-125.0))
    j = (x + f32(12582912.0)).astype(f32)
    f = (x - (j - f32(12582912.0))).astype(f32)
    fma = lambda a, b, c: (a.astype(np.float64) * b + c).astype(f32)   # one rounding, like FFMA
    p = fma(np.full_like(f, c2), f, c1)
    p = fma(p, f, c0)
    bits = p.view(np.int32) + (j.view(np.int32) << 23)
    return bits.view(f32).astype(np.float64)


def test_deg2_relative_error_below_a_thirtieth_of_e4m3_half_step():
    # the 8-bit softmax's arguments lie in [-inf, 2 + log2(224)]; e4m3's half step is 2^-4
    x = np.concatenate([np.linspace(-125, 9, 400001), np.random.default_rng(1).uniform(-30, 9, 200000)])
    x32 = x.astype(np.float32).astype(np.float64)
    rel = np.abs(emulate_deg2(x32) / np.exp2(x32) - 1)
    assert rel.max() <= 1.8e-3, rel.max()
    assert rel.max() * 30 < 2.0 ** -4


def test_deg2_clamp_keeps_results_tiny_and_positive():
    y = emulate_deg2(np.array([-np.inf, -1000.0, -125.0], dtype=np.float64))
    assert np.all(y > 0) and np.all(y < 2.0 ** -124)


def test_deg2_coefficients_are_the_fitted_ones():
    from video_dit_full_b200.fit_exp2_poly import fit
    np.testing.assert_allclose(header_coefficients_deg2(), fit(2), rtol=1e-6)
