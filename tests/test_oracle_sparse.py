"""Pins of the block-sparse attention oracle (oracle/block_sparse.py), CPU only.

* brute force: pure-Python masked softmax attention (math.fsum, exp(s)/sum exp(s))
  on tiny inputs with ragged last blocks and rows whose blocks allow nothing;
* block-diagonal masks reduce to the dense oracle on each 64-token slice;
* an all-ones mask is the dense oracle; no allowed key gives o = 0, lse = -inf;
* permuting the keys (with their values) inside an allowed block changes nothing.
"""
import itertools
import math

import numpy as np
import pytest

import oracle
import synth
from oracle import block_sparse as bs


def rand(shape, seed, scale=0.7):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def brute(q, k, v, mask):
    B, Sq, H, D = q.shape
    Sk = k.shape[1]
    o = np.zeros((B, Sq, H, D))
    lse = np.full((B, H, Sq), -np.inf)
    for b, h, i in itertools.product(range(B), range(H), range(Sq)):
        keys = [j for j in range(Sk) if mask[b, h, i // 64, j // 64]]
        if not keys:
            continue
        sc = [math.fsum(float(q[b, i, h, d]) * float(k[b, j, h, d]) for d in range(D)) / math.sqrt(D) for j in keys]
        w = [math.exp(s) for s in sc]
        z = math.fsum(w)
        for d in range(D):
            o[b, i, h, d] = math.fsum(wj * float(v[b, j, h, d]) for wj, j in zip(w, keys)) / z
        lse[b, h, i] = math.log(z)
    return o, lse


@pytest.mark.parametrize("Sq,Sk,D", [(70, 130, 4), (129, 65, 8), (5, 200, 4)])
def test_brute_force_with_empty_rows(Sq, Sk, D):
    B, H = 1, 2
    q, k, v = rand((B, Sq, H, D), 1), rand((B, Sk, H, D), 2), rand((B, Sk, H, D), 3)
    mask = synth.block_mask(B, H, bs.blocks(Sq), bs.blocks(Sk), 0.5, seed=Sq)
    mask[0, 1, 0, :] = 0                                    # query block 0 of head 1 sees nothing
    o, lse = bs.attn_fwd_block_sparse(q, k, v, mask)
    ob, lb = brute(q, k, v, mask)
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lb, rtol=1e-12, atol=1e-13)
    assert np.all(o[0, :64, 1] == 0) and np.all(np.isneginf(lse[0, 1, :64]))


def test_block_diagonal_mask_is_dense_attention_per_block():
    B, H, D, S = 1, 2, 8, 64 * 3 + 17
    q, k, v = rand((B, S, H, D), 4), rand((B, S, H, D), 5), rand((B, S, H, D), 6)
    nb = bs.blocks(S)
    mask = np.zeros((B, H, nb, nb), dtype=np.uint8)
    for i in range(nb):
        mask[:, :, i, i] = 1
    o, lse = bs.attn_fwd_block_sparse(q, k, v, mask)
    for i in range(nb):
        sl = slice(64 * i, min(S, 64 * i + 64))
        od, ld = oracle.attn_fwd(q[:, sl], k[:, sl], v[:, sl])
        np.testing.assert_allclose(o[:, sl], od, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lse[:, :, sl], ld, rtol=1e-12, atol=1e-14)


def test_all_ones_is_dense_and_row_subsets():
    B, H, D, S = 2, 2, 8, 150
    q, k, v = rand((B, S, H, D), 7), rand((B, S, H, D), 8), rand((B, S, H, D), 9)
    mask = np.ones((B, H, 3, 3), dtype=np.uint8)
    o, lse = bs.attn_fwd_block_sparse(q, k, v, mask)
    od, ld = oracle.attn_fwd(q, k, v)
    np.testing.assert_allclose(o, od, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, ld, rtol=1e-12, atol=1e-14)
    rows = np.array([0, 63, 64, 149])
    o2, l2 = bs.attn_fwd_block_sparse(q, k, v, mask, rows=rows, heads=[1])
    np.testing.assert_allclose(o2, o[:, rows][:, :, [1]], rtol=1e-13)


def test_key_permutation_inside_an_allowed_block():
    B, H, D, S = 1, 1, 8, 128
    q, k, v = rand((B, S, H, D), 10), rand((B, S, H, D), 11), rand((B, S, H, D), 12)
    mask = np.array([[[[1, 0], [1, 1]]]], dtype=np.uint8)
    perm = np.concatenate([np.random.default_rng(0).permutation(64), 64 + np.arange(64)])
    o1, l1 = bs.attn_fwd_block_sparse(q, k, v, mask)
    o2, l2 = bs.attn_fwd_block_sparse(q, k[:, perm], v[:, perm], mask)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-14)


def test_mask_generator_keeps_the_stated_count():
    m = synth.block_mask(2, 3, 5, 16, 0.125, seed=1)
    assert m.shape == (2, 3, 5, 16) and np.all(m.sum(axis=3) == 2)
    assert synth.block_mask(1, 1, 2, 3, 0.01).sum(axis=3).min() == 1
