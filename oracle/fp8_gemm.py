"""FP8 GEMM of the DiT linear layers: the oracle of the quantisers and the product.

TEST INFRASTRUCTURE ONLY (same rule as ``oracle.attention``): only tests,
``__graft_entry__.smoke()`` and the bench's CPU-baseline leg use it.

The pages: kwkr.cn Wan explainer, section 4.2 (the most expensive matrix
multiplications run in FP8; weights are quantised per tensor, activations per
token, almost losslessly), and the Wan 2.1 paper-podcast summary, section
"干预与形式化" (FP8 GEMM, 1.13x).  Readings where the pages give no formula:
e4m3 codes (largest finite 448), absmax scaling so that the largest magnitude of
each token (row of X) and of the whole weight maps to 448, round to nearest
even, fp32 accumulation, bf16 output, no bias.

For X [M, K] (tokens x in-features) and W [N, K] (out-features x in-features):
    sx[m] = fp32(absmax_k |X[m, k]| / 448),  inv_x[m] = fp32(448 / absmax_k |X[m, k]|)
    xq[m, k] = e4m3(fp32(X[m, k] * inv_x[m]))                      (1 and 1 for a zero row)
    sw = fp32(absmax |W| / 448),             wq = e4m3(fp32(W * fp32(448 / absmax |W|)))
    Y[m, n] = sx[m] * sw * sum_k xq[m, k] wq[n, k]                  (exact, fp64 here)
The scale and the scaled value that decide a code are fp32 operations, the
same ones the CUDA quantisers perform, so codes compare bit for bit.
"""
from __future__ import annotations

import numpy as np

from .quant8 import e4m3_bits, e4m3_round

E4M3_MAX = 448.0


def _f32(x) -> np.ndarray:
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32)
    return x.astype(np.float32)


def _codes(xf: np.ndarray, amax: np.ndarray):
    """fp32 values and fp32 absmax (broadcastable) -> (e4m3 bits, e4m3 values, fp32 scale)."""
    zero = amax == 0
    safe = np.where(zero, np.float32(1.0), amax).astype(np.float32)
    inv = np.where(zero, np.float32(1.0), np.float32(E4M3_MAX) / safe).astype(np.float32)
    scale = np.where(zero, np.float32(1.0), safe / np.float32(E4M3_MAX)).astype(np.float32)
    quot = (xf * inv).astype(np.float32)
    return e4m3_bits(quot), e4m3_round(quot), scale


def quant_rows(x):
    """Per-token quantiser of X [M, K]: (codes uint8 [M, K], values fp64 [M, K], sx fp32 [M])."""
    xf = _f32(x)
    amax = np.abs(xf).max(axis=1).astype(np.float32)
    bits, vals, scale = _codes(xf, amax[:, None])
    return bits, vals, scale[:, 0]


def quant_tensor(w):
    """Per-tensor quantiser of W [N, K]: (codes uint8 [N, K], values fp64 [N, K], sw fp32)."""
    wf = _f32(w)
    amax = np.float32(np.abs(wf).max())
    bits, vals, scale = _codes(wf, np.asarray(amax, dtype=np.float32))
    return bits, vals, np.float32(scale)


def gemm_from_codes(xv, sx, wv, sw, rows=None):
    """Y = diag(sx) (xq wq^T) sw in fp64 from the code values; `rows` picks rows of X."""
    xv = np.asarray(xv, dtype=np.float64)
    sx = np.asarray(sx, dtype=np.float64)
    if rows is not None:
        xv, sx = xv[rows], sx[rows]
    return (xv @ np.asarray(wv, dtype=np.float64).T) * sx[:, None] * float(sw)


def fp8_linear(x, w, rows=None):
    """The whole recipe on bf16 (or float) X and W: fp64 Y [M or len(rows), N]."""
    _, xv, sx = quant_rows(x)
    _, wv, sw = quant_tensor(w)
    return gemm_from_codes(xv, sx, wv, sw, rows)


__all__ = ["quant_rows", "quant_tensor", "gemm_from_codes", "fp8_linear", "E4M3_MAX"]
