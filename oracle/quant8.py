"""Quantisers of the 8-bit attention recipe, and an fp64 simulation of it.

TEST INFRASTRUCTURE ONLY (same rule as ``oracle.attention``): only tests,
``__graft_entry__.smoke()`` and the bench's CPU-baseline leg use it.

The pages' 8-bit FlashAttention: Wan 2.1 paper-podcast summary, section
"干预与形式化" (mixed int8/FP8 with FP32 accumulation across blocks, 1.27x,
95% MFU on H20) and the kwkr.cn Wan explainer, section 4.2 (FlashAttention3
8-bit: INT8 for Q, K, V, FP8 output, FP32 register accumulation).  The two
disagree on which operands are int8; the reading taken here is int8 Q and K,
e4m3 P and V, per-(batch, head, 64-token block) scales (absmax/127 for int8;
for V the smallest power of two >= absmax/448), each block's V scale folded
into P before P is quantised (an exact power-of-two factor), and all blocks'
P.V products summed by one fp32 accumulation.

Where a floating-point value decides a code (the scale, the scaled value and
its rounding), the computation is done in fp32 exactly as the CUDA quantiser
does it, so codes can be compared bit for bit:
    scale = fp32(absmax / 127), codes from fp32(x * fp32(127 / absmax))   (int8)
    scale = max(smallest power of two >= fp32(absmax / 448), 2^-126)   (e4m3)
    scale = 1 when absmax == 0
    int8 code = clamp(rint_even(fp32(x * fp32(127 / absmax))), -127, 127)
    e4m3 code = e4m3_rne_satfinite(x / scale)        (exact: scale is a power of two)

The unquantised fp64 oracle (``oracle.attention.attn_fwd``) is what the 8-bit
path's parity is judged against; ``attn_fwd_q8_sim`` is a diagnostic only.
"""
from __future__ import annotations

import numpy as np

from .attention import widen

BLOCK = 64
E4M3_MAX = 448.0


def _f32(x) -> np.ndarray:
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32)
    return x.astype(np.float32)


def e4m3_round(x) -> np.ndarray:
    """Round to the nearest FP8 E4M3 (fn variant: bias 7, 3 mantissa bits,
    largest finite 448, no infinities) with ties to even, saturating finite
    values beyond 448 to +-448.  Returns the rounded values as fp64.

    Representable magnitudes: 0, (f/8)*2^-6 for f = 1..7 (subnormal), and
    (1 + f/8)*2^(E-7) for E = 1..15, f = 0..7 except E = 15, f = 7 (NaN).
    """
    a = np.abs(np.asarray(x, dtype=np.float64))
    _, ex = np.frexp(a)                 # a = mant * 2^ex, mant in [0.5, 1)
    e = np.maximum(ex - 1, -6)          # binade exponent; subnormals share 2^-6's quantum
    quantum = np.ldexp(1.0, e - 3)
    r = np.rint(a / quantum) * quantum  # exact division by a power of two; rint = ties-to-even
    r = np.where(a >= E4M3_MAX, E4M3_MAX, np.minimum(r, E4M3_MAX))
    return np.copysign(r, x)


def e4m3_bits(x) -> np.ndarray:
    """The E4M3 bit pattern (uint8) of ``e4m3_round(x)``."""
    r = e4m3_round(x)
    sign = (np.signbit(r)).astype(np.uint8) << 7
    a = np.abs(r)
    _, ex = np.frexp(a)
    E = np.where(a < 2.0 ** -6, 0, ex - 1 + 7)
    frac = np.where(E == 0, a / 2.0 ** -9, (a / np.ldexp(1.0, E - 7) - 1.0) * 8.0)
    return (sign | (E.astype(np.uint8) << 3) | np.rint(frac).astype(np.uint8)).astype(np.uint8)


def block_absmax(x: np.ndarray, block: int = BLOCK) -> np.ndarray:
    """absmax over each (b, h, 64-token block) of [B, S, H, D] fp32 values -> [B, H, nblk] fp32."""
    B, S, H, D = x.shape
    nb = (S + block - 1) // block
    out = np.zeros((B, H, nb), dtype=np.float32)
    a = np.abs(x)
    for t in range(nb):
        out[:, :, t] = a[:, t * block:(t + 1) * block].max(axis=(1, 3))
    return out


def quant_int8(x, block: int = BLOCK):
    """int8 codes [B, S, H, D] and fp32 scales [B, H, nblk] of Q or K.

    scale = fp32(absmax / 127) dequantises; the codes are rint(fp32(x * fp32(127 / absmax)))."""
    xf = _f32(x)
    amax = block_absmax(xf, block)
    scale = np.where(amax == 0, np.float32(1.0), amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(amax == 0, np.float32(1.0), amax).astype(np.float32)
    inv = np.where(amax == 0, np.float32(1.0), np.float32(127.0) / safe).astype(np.float32)
    per_tok = np.repeat(inv, block, axis=2)[:, :, : xf.shape[1]]            # [B, H, S]
    quot = (xf * per_tok.transpose(0, 2, 1)[:, :, :, None]).astype(np.float32)
    codes = np.clip(np.rint(quot), -127, 127).astype(np.int8)
    return codes, scale


def pow2_ceil_f32(q: np.ndarray) -> np.ndarray:
    """The smallest power of two >= q (q > 0, fp32), exactly: q itself when q is one."""
    mant, ex = np.frexp(q.astype(np.float32))            # q = mant * 2^ex, mant in [0.5, 1)
    return np.where(mant == 0.5, q, np.ldexp(np.float32(1.0), ex)).astype(np.float32)


def quant_e4m3(x, block: int = BLOCK):
    """E4M3 codes (uint8 bit patterns) [B, S, H, D], their values (fp64) and fp32 scales [B, H, nblk] of V.

    Each block's scale is the smallest power of two >= fp32(absmax / 448), at
    least 2^-126 (1 for an all-zero block): the codes then span up to 448 and any
    two blocks' scales differ by an exact power of two."""
    xf = _f32(x)
    amax = block_absmax(xf, block)
    q = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    scale = np.where(amax == 0, np.float32(1.0), pow2_ceil_f32(np.where(amax == 0, np.float32(1.0), q)))
    scale = np.maximum(scale, np.float32(2.0 ** -126)).astype(np.float32)   # always a normal float
    per_tok = np.repeat(scale, block, axis=2)[:, :, : xf.shape[1]]
    quot = (xf / per_tok.transpose(0, 2, 1)[:, :, :, None]).astype(np.float32)
    return e4m3_bits(quot), e4m3_round(quot), scale


def _fold_factor(sv_bh: np.ndarray, S: int, block: int) -> np.ndarray:
    """Per key j of one (b, h): sV(t(j)) / sV_max, the power-of-two factor that carries the
    key's 64-token block scale into P in the folded form of the recipe."""
    sv_key = np.repeat(sv_bh, block)[:S].astype(np.float64)
    return sv_key / float(sv_bh.max())


def attn_fwd_q8_sim(q, k, v, rows=None, heads=None, block: int = BLOCK):
    """Diagnostic fp64 simulation of the 8-bit recipe in its folded form.

    Scores from the int8 codes, s_ij = (q8_i . k8_j) sQ(i) sK(j) / sqrt(D);
    p_ij = exp(s_ij - max_j s_ij) in [0, 1]; l_i = sum_j p_ij (unquantised).
    Each 64-key block t's V scale is folded into P before P is quantised,
    P8_ij = e4m3(448 p_ij sV(t) / sV_max) with sV_max the largest block scale
    of the (b, h), so one fp32 accumulation carries every block:
    o_i = (sum_j P8_ij v8_j) * sV_max / 448 / l_i.

    Pinned against ``attn_fwd_q8_blockwise`` (the per-block accumulation form):
    the two are equal wherever no P code is subnormal, since the fold factor is
    an exact power of two."""
    B, S, H, D = q.shape
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    heads = list(range(H)) if heads is None else list(heads)
    q8, sq = quant_int8(q, block)
    k8, sk = quant_int8(k, block)
    _, v8, sv = quant_e4m3(v, block)
    o = np.empty((B, len(rows), len(heads), D))
    lse = np.empty((B, len(heads), len(rows)))
    for b in range(B):
        for hi, h in enumerate(heads):
            Q = q8[b, rows, h, :].astype(np.float64) * sq[b, h, rows // block][:, None].astype(np.float64)
            Kd = k8[b, :, h, :].astype(np.float64) * np.repeat(sk[b, h], block)[:S, None].astype(np.float64)
            s = (Q @ Kd.T) / np.sqrt(D)
            m = s.max(axis=1)
            p = np.exp(s - m[:, None])
            l = p.sum(axis=1)
            sv_max = float(sv[b, h].max())
            p8 = e4m3_round(p * (E4M3_MAX * _fold_factor(sv[b, h], S, block))[None, :])
            o[b, :, hi, :] = (p8 @ v8[b, :, h, :]) * (sv_max / E4M3_MAX) / l[:, None]
            lse[b, hi] = m + np.log(l)
    return o, lse


def attn_fwd_q8_blockwise(q, k, v, rows=None, heads=None, block: int = BLOCK):
    """The 8-bit recipe with its cross-block accumulation written out block by block.

    Wan 2.1 paper-podcast summary, section "干预与形式化" (8-bit FlashAttention:
    per-block quantised operands, FP32 accumulation across blocks) and the kwkr.cn
    Wan explainer, section 4.2.  For one query row i and each 64-key block t in turn:
      scores   s_ij = (q8_i . k8_j) sQ(i) sK(t) / sqrt(D)        for j in block t
      weights  p_ij = exp(s_ij - m_i), m_i the row's maximum over all keys
      P codes  e4m3(448 p_ij)                 (P's own block scale: 1/448)
      product  O_t = sum_{j in t} e4m3(448 p_ij) v8_j        (the block's 8-bit MMA)
      add      acc += O_t * sV(t) / 448       (dequantised, accumulated across blocks)
    and o_i = acc / l_i with l_i = sum_j p_ij (unquantised), lse_i = m_i + ln l_i.
    No scale is folded into P here, so this form shares no step with the folded
    simulation beyond the quantisers."""
    B, S, H, D = q.shape
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    heads = list(range(H)) if heads is None else list(heads)
    q8, sq = quant_int8(q, block)
    k8, sk = quant_int8(k, block)
    _, v8, sv = quant_e4m3(v, block)
    nb = (S + block - 1) // block
    o = np.empty((B, len(rows), len(heads), D))
    lse = np.empty((B, len(heads), len(rows)))
    for b in range(B):
        for hi, h in enumerate(heads):
            Qd = q8[b, rows, h, :].astype(np.float64) * sq[b, h, rows // block][:, None].astype(np.float64)
            s_blocks = []
            for t in range(nb):
                kt = k8[b, t * block:(t + 1) * block, h, :].astype(np.float64) * float(sk[b, h, t])
                s_blocks.append((Qd @ kt.T) / np.sqrt(D))
            m = np.max([sb.max(axis=1) for sb in s_blocks], axis=0)
            acc = np.zeros((len(rows), D))
            l = np.zeros(len(rows))
            for t in range(nb):
                p = np.exp(s_blocks[t] - m[:, None])
                l += p.sum(axis=1)
                o_t = e4m3_round(E4M3_MAX * p) @ v8[b, t * block:(t + 1) * block, h, :]
                acc += o_t * (float(sv[b, h, t]) / E4M3_MAX)
            o[b, :, hi, :] = acc / l[:, None]
            lse[b, hi] = m + np.log(l)
    return o, lse


__all__ = ["e4m3_round", "e4m3_bits", "quant_int8", "quant_e4m3", "attn_fwd_q8_sim", "attn_fwd_q8_blockwise",
           "block_absmax", "widen", "BLOCK"]
