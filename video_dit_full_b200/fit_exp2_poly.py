"""Fit the polynomial the kernels use for 2^f on [-1/2, 1/2].

    python -m video_dit_full_b200.fit_exp2_poly

Minimax in relative error, by the Lawson iteration (iteratively reweighted
least squares, which converges to the Chebyshev/minimax solution) on a dense
grid.  Prints the coefficients c0..cN (2^f ~ sum c_k f^k) and the maximum
relative error, both in fp64 and with the coefficients rounded to fp32 and
the polynomial evaluated in fp32 Horner form as the kernel does.
"""
from __future__ import annotations

import argparse

import numpy as np


def fit(degree: int, iters: int = 400, n: int = 20001):
    f = np.linspace(-0.5, 0.5, n)
    y = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / y[:, None]    # relative error: (p - y) / y
    rhs = np.ones_like(f)
    w = np.full(n, 1.0 / n)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], rhs * sw, rcond=None)
        err = np.abs(A @ c - rhs)
        w = w * err
        w /= w.sum()
    return c


def eval_fp32(c, f):
    c32 = np.asarray(c, dtype=np.float32)
    f32 = np.asarray(f, dtype=np.float32)
    p = np.full_like(f32, c32[-1])
    for ck in c32[-2::-1]:
        p = (p * f32 + ck).astype(np.float32)          # the kernel uses FFMA (one rounding); close enough here
    return p.astype(np.float64)


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--degree", type=int, default=3)
    a = ap.parse_args()
    c = fit(a.degree)
    f = np.linspace(-0.5, 0.5, 200001)
    rel64 = np.abs(np.polyval(c[::-1], f) / np.exp2(f) - 1).max()
    rel32 = np.abs(eval_fp32(c, f) / np.exp2(f) - 1).max()
    print("coefficients (c0..cN):", ", ".join(repr(float(np.float32(x))) for x in c))
    print(f"max relative error: fp64 {rel64:.3e}, fp32 coefficients {rel32:.3e}")
