"""Pins of the fp64 oracle for queries and keys of different lengths (cross-attention), CPU only.

The DiT block's cross-attention takes its queries from the Sq video tokens and
its keys/values from the Sk = 512 tokens of the umT5 text embedding (Wan 2.1
paper-podcast summary, section "干预与形式化").  The definition is the same as
self-attention with the key index running over [0, Sk):

* brute force: a pure-Python formulation (math.fsum, exp(s)/sum exp(s) without
  max subtraction) on tiny Sq != Sk inputs;
* closed forms: Sk = 1 (every query returns v_0, lse_i = q_i.k_0/sqrt(D)),
  Q = 0 (mean of the Sk values, lse = ln Sk), and the backward with Sk = 1
  (dQ = dK = 0, dV_0 = sum over every query of dO_i);
* backward: central finite differences of f = sum(O * dO) with Sq != Sk,
  sum_j dK_j = 0, sampled key rows equal the full computation.
"""
import itertools
import math

import numpy as np
import pytest

import oracle
from oracle import attention as oa


def rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def brute_cross(q, k, v):
    B, Sq, H, D = q.shape
    Sk = k.shape[1]
    o = np.zeros((B, Sq, H, D))
    lse = np.zeros((B, H, Sq))
    for b, h, i in itertools.product(range(B), range(H), range(Sq)):
        sc = [math.fsum(float(q[b, i, h, d]) * float(k[b, j, h, d]) for d in range(D)) / math.sqrt(D)
              for j in range(Sk)]
        w = [math.exp(s) for s in sc]
        z = math.fsum(w)
        for d in range(D):
            o[b, i, h, d] = math.fsum(w[j] * float(v[b, j, h, d]) for j in range(Sk)) / z
        lse[b, h, i] = math.log(z)
    return o, lse


@pytest.mark.parametrize("Sq,Sk,D,B,H", [(1, 3, 4, 1, 1), (5, 2, 8, 1, 2), (3, 17, 4, 2, 1),
                                         (17, 5, 128, 1, 1), (9, 1, 8, 1, 2)])
def test_brute_force_cross_forward(Sq, Sk, D, B, H):
    q = rand((B, Sq, H, D), 1, 0.7)
    k, v = rand((B, Sk, H, D), 2, 0.7), rand((B, Sk, H, D), 3, 0.7)
    o, lse = oracle.attn_fwd(q, k, v)
    assert o.shape == (B, Sq, H, D) and lse.shape == (B, H, Sq)
    ob, lb = brute_cross(q, k, v)
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lb, rtol=1e-12, atol=1e-13)


def test_single_key_every_query_returns_it():
    q = rand((1, 7, 2, 16), 4)
    k, v = rand((1, 1, 2, 16), 5), rand((1, 1, 2, 16), 6)
    o, lse = oracle.attn_fwd(q, k, v)
    np.testing.assert_allclose(o, np.broadcast_to(v, o.shape), rtol=1e-15)
    for h in range(2):
        np.testing.assert_allclose(lse[0, h], q[0, :, h] @ k[0, 0, h] / 4.0, rtol=1e-13)


def test_zero_query_averages_the_keys_values():
    q = np.zeros((1, 4, 2, 8))
    k, v = rand((1, 11, 2, 8), 7), rand((1, 11, 2, 8), 8)
    o, lse = oracle.attn_fwd(q, k, v)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=1, keepdims=True), o.shape), rtol=1e-13)
    np.testing.assert_allclose(lse, math.log(11), rtol=1e-15)


def _f(q, k, v, do):
    o, _ = oracle.attn_fwd(q, k, v)
    return float((o * do).sum())


@pytest.mark.parametrize("Sq,Sk,D", [(5, 3, 3), (2, 6, 4)])
def test_cross_backward_finite_differences(Sq, Sk, D):
    B, H = 1, 2
    q, do = rand((B, Sq, H, D), 31), rand((B, Sq, H, D), 34)
    k, v = rand((B, Sk, H, D), 32), rand((B, Sk, H, D), 33)
    g = oracle.attn_bwd(q, k, v, do)
    assert g["dq"].shape == q.shape and g["dk"].shape == k.shape and g["dv"].shape == v.shape
    eps = 1e-6
    for name, x, grad in (("q", q, g["dq"]), ("k", k, g["dk"]), ("v", v, g["dv"])):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            fp = _f(args["q"], args["k"], args["v"], do)
            args[name] = xm
            fm = _f(args["q"], args["k"], args["v"], do)
            fd[idx] = (fp - fm) / (2 * eps)
        rel = np.linalg.norm(grad - fd) / np.linalg.norm(fd)
        assert rel < 1e-6, (name, rel)


def test_cross_backward_single_key_closed_form():
    q, do = rand((1, 6, 2, 8), 35), rand((1, 6, 2, 8), 38)
    k, v = rand((1, 1, 2, 8), 36), rand((1, 1, 2, 8), 37)
    g = oracle.attn_bwd(q, k, v, do)
    np.testing.assert_allclose(g["dq"], 0.0, atol=1e-15)
    np.testing.assert_allclose(g["dk"], 0.0, atol=1e-14)
    np.testing.assert_allclose(g["dv"][:, 0], do.sum(axis=1), rtol=1e-14)


def test_cross_backward_sum_dk_vanishes_and_sampled_rows_match(monkeypatch):
    q, do = rand((1, 23, 3, 8), 39), rand((1, 23, 3, 8), 42)
    k, v = rand((1, 9, 3, 8), 40), rand((1, 9, 3, 8), 41)
    full = oracle.attn_bwd(q, k, v, do)
    assert full["dk"].shape == (1, 9, 3, 8) and full["lse"].shape == (1, 3, 23)
    scale = np.abs(full["dk"]).max()
    np.testing.assert_allclose(full["dk"].sum(axis=1), 0.0, atol=1e-13 * scale * 9)
    monkeypatch.setattr(oa, "ROW_CHUNK", 4)
    qr, kr, heads = np.array([0, 5, 22]), np.array([0, 8]), [0, 2]
    part = oracle.attn_bwd(q, k, v, do, q_rows=qr, k_rows=kr, heads=heads)
    np.testing.assert_allclose(part["dq"], full["dq"][:, qr][:, :, heads], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(part["dk"], full["dk"][:, kr][:, :, heads], rtol=1e-11, atol=1e-15)
    np.testing.assert_allclose(part["dv"], full["dv"][:, kr][:, :, heads], rtol=1e-12, atol=1e-15)
