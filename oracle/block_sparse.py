"""Block-sparse attention with a given 64 x 64 block mask: the oracle.

TEST INFRASTRUCTURE ONLY (same rule as ``oracle.attention``).

The pages: the FastWan / VSA article on the first page ("一夜颠覆Sora神话，H200单卡
5秒出片…"): video sparse attention keeps, for each 64-token query block, a subset
of the 64-token key blocks (87.5 % sparsity in its scaling runs), and compares its
kernel with FlexAttention running the same block-sparse mask of 64 x 64 blocks.
Here the mask is given (the learned coarse stage that picks the blocks is not
built).  Readings: block b of a sequence holds tokens [64 b, 64 b + 64) (the last
block may be short); mask[b, h, i, j] = 1 lets query block i attend key block j;
a query row whose blocks allow no key has o = 0 and lse = -inf.

For each (b, h) and query row r in block i = r // 64:
    allowed(r) = { keys c : mask[b, h, i, c // 64] = 1 }
    s_rc = (q_r . k_c) / sqrt(D) over allowed(r)
    lse_r = ln sum_{c in allowed(r)} exp(s_rc)
    o_r   = sum_{c in allowed(r)} exp(s_rc - lse_r) v_c
"""
from __future__ import annotations

import numpy as np

from .attention import widen

BLOCK = 64


def blocks(n: int) -> int:
    return (n + BLOCK - 1) // BLOCK


def attn_fwd_block_sparse(q, k, v, mask, rows=None, heads=None):
    """q [B, Sq, H, D], k, v [B, Sk, H, D], mask uint8 [B, H, ceil(Sq/64), ceil(Sk/64)].
    Returns (o [B, R, Hs, D] fp64, lse [B, Hs, R] fp64) for the chosen rows and heads."""
    B, Sq, H, D = q.shape
    Sk = k.shape[1]
    mask = np.asarray(mask)
    if mask.shape != (B, H, blocks(Sq), blocks(Sk)):
        raise ValueError(f"mask shape {mask.shape}, expected {(B, H, blocks(Sq), blocks(Sk))}")
    rows = np.arange(Sq) if rows is None else np.asarray(rows, dtype=np.int64)
    heads = list(range(H)) if heads is None else list(heads)
    scale = 1.0 / np.sqrt(D)
    key_block = np.arange(Sk) // BLOCK
    o = np.zeros((B, len(rows), len(heads), D))
    lse = np.full((B, len(heads), len(rows)), -np.inf)
    for b in range(B):
        for hi, h in enumerate(heads):
            K, V = widen(k[b, :, h, :]), widen(v[b, :, h, :])
            Q = widen(q[b, rows, h, :])
            allowed = mask[b, h][rows // BLOCK][:, key_block] != 0          # [R, Sk]
            s = np.where(allowed, (Q @ K.T) * scale, -np.inf)
            any_ok = allowed.any(axis=1)
            m = np.where(any_ok, s.max(axis=1), 0.0)
            e = np.exp(s - m[:, None])                                       # 0 where not allowed
            l = e.sum(axis=1)
            ok = any_ok
            o[b, ok, hi, :] = (e[ok] @ V) / l[ok, None]
            lse[b, hi, ok] = m[ok] + np.log(l[ok])
    return o, lse


__all__ = ["attn_fwd_block_sparse", "blocks", "BLOCK"]
