"""Pins of the fp64 oracle to things other than itself (CPU only).

* brute force: a second formulation in pure Python (math.fsum, softmax as
  exp(s)/sum exp(s) without max subtraction, division by the sum) on tiny inputs;
* closed forms: S = 1, S = 2 (logistic weights), Q = 0 (mean of V, lse = ln S);
* invariants: rows of P sum to 1, constant V, joint K/V permutation, Q row
  permutation, a dominant key, shift of all keys by one vector;
* backward: central finite differences of f = sum(O * dO), S = 1 closed form,
  sum_j dK_j = 0, sum_j dS_ij = 0, sampled rows equal the full computation;
* planted mistakes: mutated copies of the oracle's row kernel fail the pins.
"""
import itertools
import math

import numpy as np
import pytest

import oracle
from oracle import attention as oa


def rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def brute_fwd(q, k, v):
    """Pure-Python fp64 attention of every (b, h, i), independent of the oracle."""
    B, S, H, D = q.shape
    o = np.zeros((B, S, H, D))
    lse = np.zeros((B, H, S))
    for b, h, i in itertools.product(range(B), range(H), range(S)):
        sc = [math.fsum(float(q[b, i, h, d]) * float(k[b, j, h, d]) for d in range(D)) / math.sqrt(D)
              for j in range(S)]
        w = [math.exp(s) for s in sc]
        z = math.fsum(w)
        for d in range(D):
            o[b, i, h, d] = math.fsum(w[j] * float(v[b, j, h, d]) for j in range(S)) / z
        lse[b, h, i] = math.log(z)
    return o, lse


@pytest.mark.parametrize("S,D,B,H", [(1, 1, 1, 1), (2, 4, 1, 2), (3, 8, 2, 1), (5, 128, 1, 1),
                                     (17, 4, 1, 2), (17, 8, 2, 2)])
def test_brute_force_forward(S, D, B, H):
    q, k, v = (rand((B, S, H, D), s, 0.7) for s in (1, 2, 3))
    o, lse = oracle.attn_fwd(q, k, v)
    ob, lb = brute_fwd(q, k, v)
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lb, rtol=1e-12, atol=1e-13)


def test_bf16_inputs_widen_exactly():
    bits = np.array([0x3F80, 0xC040, 0x0000, 0x3E00, 0x7F7F], dtype=np.uint16)
    np.testing.assert_array_equal(oracle.widen(bits), [1.0, -3.0, 0.0, 0.125, 3.3895313892515355e38])


def test_closed_form_single_key():
    q, k, v = rand((1, 1, 2, 16), 4), rand((1, 1, 2, 16), 5), rand((1, 1, 2, 16), 6)
    o, lse = oracle.attn_fwd(q, k, v)
    np.testing.assert_allclose(o, v, rtol=1e-15)
    np.testing.assert_allclose(lse[0, :, 0], (q[0, 0] * k[0, 0]).sum(-1) / 4.0, rtol=1e-14)


def test_closed_form_two_keys():
    q, k, v = rand((1, 2, 1, 8), 7), rand((1, 2, 1, 8), 8), rand((1, 2, 1, 8), 9)
    o, _ = oracle.attn_fwd(q, k, v)
    for i in range(2):
        s0 = q[0, i, 0] @ k[0, 0, 0] / math.sqrt(8)
        s1 = q[0, i, 0] @ k[0, 1, 0] / math.sqrt(8)
        w0 = 1.0 / (1.0 + math.exp(s1 - s0))
        np.testing.assert_allclose(o[0, i, 0], w0 * v[0, 0, 0] + (1 - w0) * v[0, 1, 0], rtol=1e-13)


def test_closed_form_zero_query():
    S = 33
    q = np.zeros((1, S, 2, 8))
    k, v = rand((1, S, 2, 8), 10), rand((1, S, 2, 8), 11)
    o, lse = oracle.attn_fwd(q, k, v)
    np.testing.assert_allclose(o[0, 5], v[0].mean(axis=0), rtol=1e-13)
    np.testing.assert_allclose(lse, math.log(S), rtol=1e-15)


def test_rows_of_p_sum_to_one():
    q, k = rand((1, 40, 1, 16), 12, 3.0), rand((1, 40, 1, 16), 13, 3.0)
    p = oracle.softmax_matrix(q, k)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-12)
    assert np.all(p >= 0)


def test_constant_v_gives_constant_output():
    q, k = rand((2, 30, 3, 16), 14), rand((2, 30, 3, 16), 15)
    v = np.broadcast_to(rand((1, 1, 3, 16), 16), (2, 30, 3, 16)).copy()
    o, _ = oracle.attn_fwd(q, k, v)
    np.testing.assert_allclose(o, v, rtol=1e-13)


def test_joint_kv_permutation_and_q_permutation():
    q, k, v = rand((1, 25, 2, 8), 17), rand((1, 25, 2, 8), 18), rand((1, 25, 2, 8), 19)
    o, lse = oracle.attn_fwd(q, k, v)
    perm = np.random.default_rng(20).permutation(25)
    o2, lse2 = oracle.attn_fwd(q, k[:, perm], v[:, perm])
    np.testing.assert_allclose(o2, o, rtol=1e-12)
    np.testing.assert_allclose(lse2, lse, rtol=1e-13)
    o3, lse3 = oracle.attn_fwd(q[:, perm], k, v)
    np.testing.assert_allclose(o3, o[:, perm], rtol=1e-13)
    np.testing.assert_allclose(lse3, lse[:, :, perm], rtol=1e-13)


def test_dominant_key_selects_its_value():
    D = 128
    q, k, v = rand((1, 20, 1, D), 21), rand((1, 20, 1, D), 22), rand((1, 20, 1, D), 23)
    i, j = 4, 11
    qi = q[0, i, 0]
    k[0, j, 0] = qi * (40.0 * math.sqrt(D) / (qi @ qi))     # s_ij = 40, the others ~ N(0, 1)
    o, _ = oracle.attn_fwd(q, k, v)
    np.testing.assert_allclose(o[0, i, 0], v[0, j, 0], atol=1e-10)


def test_shifting_every_key_shifts_lse_only():
    q, k, v = rand((1, 19, 2, 8), 24, 4.0), rand((1, 19, 2, 8), 25, 4.0), rand((1, 19, 2, 8), 26)
    u = rand((1, 1, 2, 8), 27, 60.0)           # scores move by q_i.u/sqrt(D), up to ~hundreds
    o, lse = oracle.attn_fwd(q, k, v)
    o2, lse2 = oracle.attn_fwd(q, k + u, v)
    np.testing.assert_allclose(o2, o, rtol=1e-9, atol=1e-12)
    shift = np.einsum("bihd,bhd->bhi", q, u[:, 0]) / math.sqrt(8)
    np.testing.assert_allclose(lse2, lse + shift, rtol=1e-12, atol=1e-9)


def test_row_and_head_subsets_and_chunking(monkeypatch):
    q, k, v = rand((2, 23, 3, 8), 28), rand((2, 23, 3, 8), 29), rand((2, 23, 3, 8), 30)
    o, lse = oracle.attn_fwd(q, k, v)
    monkeypatch.setattr(oa, "ROW_CHUNK", 4)
    rows, heads = np.array([0, 5, 6, 21, 22]), [2, 0]
    o2, lse2 = oracle.attn_fwd(q, k, v, rows=rows, heads=heads)
    np.testing.assert_allclose(o2, o[:, rows][:, :, heads], rtol=1e-14)
    np.testing.assert_allclose(lse2, lse[:, heads][:, :, rows], rtol=1e-14)


# ------------------------------- backward ---------------------------------
def _f(q, k, v, do):
    o, _ = oracle.attn_fwd(q, k, v)
    return float((o * do).sum())


@pytest.mark.parametrize("S,D", [(4, 3), (6, 5)])
def test_backward_finite_differences(S, D):
    B, H = 1, 2
    q, k, v, do = (rand((B, S, H, D), s) for s in (31, 32, 33, 34))
    g = oracle.attn_bwd(q, k, v, do)
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


def test_backward_single_key_closed_form():
    q, k, v, do = (rand((1, 1, 2, 8), s) for s in (35, 36, 37, 38))
    g = oracle.attn_bwd(q, k, v, do)
    np.testing.assert_allclose(g["dq"], 0.0, atol=1e-15)
    np.testing.assert_allclose(g["dk"], 0.0, atol=1e-15)
    np.testing.assert_allclose(g["dv"], do, rtol=1e-15)


def test_backward_sum_dk_and_ds_rows_vanish():
    q, k, v, do = (rand((1, 30, 2, 8), s) for s in (39, 40, 41, 42))
    g = oracle.attn_bwd(q, k, v, do)
    scale = np.abs(g["dk"]).max()
    np.testing.assert_allclose(g["dk"].sum(axis=1), 0.0, atol=1e-13 * scale * 30)
    # sum_j dS_ij = sum_j P_ij dP_ij - Dl_i = 0
    for h in range(2):
        p = oracle.softmax_matrix(q, k, 0, h)
        dp = do[0, :, h] @ v[0, :, h].T
        dl = (p * dp).sum(axis=1)
        np.testing.assert_allclose(dl, g["dl"][0, h], rtol=1e-12, atol=1e-14)
        ds = p * (dp - g["dl"][0, h][:, None])
        np.testing.assert_allclose(ds.sum(axis=1), 0.0, atol=1e-13)


def test_backward_sampled_rows_match_full(monkeypatch):
    q, k, v, do = (rand((1, 21, 3, 8), s) for s in (43, 44, 45, 46))
    full = oracle.attn_bwd(q, k, v, do)
    monkeypatch.setattr(oa, "ROW_CHUNK", 5)
    qr, kr, heads = np.array([0, 3, 20]), np.array([1, 19, 20]), [1, 2]
    part = oracle.attn_bwd(q, k, v, do, q_rows=qr, k_rows=kr, heads=heads)
    np.testing.assert_allclose(part["dq"], full["dq"][:, qr][:, :, heads], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(part["dk"], full["dk"][:, kr][:, :, heads], rtol=1e-11, atol=1e-15)
    np.testing.assert_allclose(part["dv"], full["dv"][:, kr][:, :, heads], rtol=1e-12, atol=1e-15)
    only_q = oracle.attn_bwd(q, k, v, do, q_rows=qr, k_rows=[], heads=heads)
    np.testing.assert_allclose(only_q["dq"], part["dq"], rtol=1e-13, atol=1e-15)
    assert only_q["dk"].shape[1] == 0


# ------------------------------ planted mistakes ---------------------------
def _mutant(kind):
    def rows_fwd(Q, K, V, scale):
        if kind == "scale_1_over_d":
            scale = scale * scale
        s = (Q @ K.T) * scale
        if kind == "keys_reversed_for_v":
            V = V[::-1]
        m = s.max(axis=1)
        lse = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
        if kind == "lse_without_max":
            lse = np.log(np.exp(s - m[:, None]).sum(axis=1))
        p = np.exp(s - lse[:, None])
        if kind == "no_normalisation":
            p = np.exp(s - m[:, None])
        return p @ V, lse
    return rows_fwd


@pytest.mark.parametrize("kind", ["scale_1_over_d", "keys_reversed_for_v", "lse_without_max",
                                  "no_normalisation"])
def test_planted_mistakes_are_caught(monkeypatch, kind):
    monkeypatch.setattr(oa, "_rows_fwd", _mutant(kind))
    q, k, v = (rand((1, 5, 1, 8), s, 1.5) for s in (47, 48, 49))
    o, lse = oracle.attn_fwd(q, k, v)
    ob, lb = brute_fwd(q, k, v)
    assert not (np.allclose(o, ob, rtol=1e-9) and np.allclose(lse, lb, rtol=1e-9))


def test_backward_by_head_threads_equal_direct_call():
    # the GPU tests' threaded per-head evaluation stacks exactly what one call returns
    from gpu_util import oracle_bwd_by_head
    x = {n: rand((2, 70, 3, 16), 40 + i) for i, n in enumerate(("q", "k", "v", "do"))}
    k_rows, q_rows = [0, 5, 69], [1, 68]
    want = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], q_rows=q_rows, k_rows=k_rows, heads=[2, 0])
    got = oracle_bwd_by_head(x, q_rows, k_rows, [2, 0], workers=2)
    for n in ("dq", "dk", "dv", "lse", "dl"):
        np.testing.assert_allclose(got[n], want[n], rtol=1e-12, atol=1e-14, err_msg=n)
