"""Parity of the cross-attention calls (wan_attn_cross_fwd / wan_attn_cross_bwd, through the
C ABI) with the fp64 oracle: video-token queries attending to Skv keys, Skv = 512 being the
umT5 text embedding's length (Wan 2.1 paper-podcast summary, section "干预与形式化").

Bars as for self-attention: O max-abs <= 1e-2 and relative Frobenius <= 5e-3 (LSE to 1e-3);
dQ, dK, dV relative Frobenius <= 2e-2.  Small key counts make the backward spread each key
tile's queries over several CTAs (fp32 reduce of dK, dV); large ones keep one CTA per key
tile: both are covered.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import bf16_to_f64, errors, inputs_for_cross, oracle_bwd_by_head, to_device

pytestmark = pytest.mark.gpu

O_MAX_ABS, O_REL_FROB, LSE_MAX_ABS, GRAD_REL_FROB = 1e-2, 5e-3, 1e-3, 2e-2
# With one key, dS = P (dP - D) vanishes in real arithmetic (P = 1, D = dO.o = dO.v = dP), so
# dQ = dK = 0.  In the kernel D is an fp32 dot product of dO with the bf16-rounded O and dP a
# tensor-core fp32 sum, |dP| ~ sqrt(D) for N(0,1) inputs: their difference is a few fp32 ulps of
# |dP| (~1e-6), and dK sums Sq of them.  1e-4 bounds that with margin; a wrong formula gives O(1).
ZERO_GRAD_ABS = 1e-4


def run_fwd(x):
    import video_dit_full_b200 as wa
    q, k, v = (to_device(x[n]) for n in "qkv")
    o, lse = wa.cross_fwd(q, k, v)
    wa.check_status()
    return o, lse


def check_fwd(x, rows=None, heads=None):
    o, lse = run_fwd(x)
    want_o, want_lse = oracle.attn_fwd(x["q"], x["k"], x["v"], rows=rows, heads=heads)
    got_o, got_lse = bf16_to_f64(o), lse.cpu().numpy().astype(np.float64)
    if rows is not None:
        got_o, got_lse = got_o[:, rows], got_lse[:, :, rows]
    if heads is not None:
        got_o, got_lse = got_o[:, :, heads], got_lse[:, heads]
    assert np.all(np.isfinite(got_o)) and np.all(np.isfinite(got_lse))
    max_abs, rel = errors(got_o, want_o)
    lse_err = float(np.abs(got_lse - want_lse).max())
    print(f"O max-abs {max_abs:.3e} rel-frob {rel:.3e}  LSE max-abs {lse_err:.3e}")
    assert max_abs <= O_MAX_ABS and rel <= O_REL_FROB, (max_abs, rel)
    assert lse_err <= LSE_MAX_ABS, lse_err
    return o, lse


@pytest.mark.parametrize("B,Sq,Skv,H", [(1, 1, 1, 1), (1, 300, 77, 2), (2, 129, 512, 1), (1, 1000, 1, 2),
                                        (1, 64, 1000, 2), (1, 257, 129, 3), (1, 1280, 512, 12)])
def test_cross_fwd_shapes_full(B, Sq, Skv, H):
    check_fwd(inputs_for_cross(B, Sq, Skv, H, seed=Sq + 7 * Skv))


def test_cross_fwd_720p_text_sampled_rows():
    w = synth.WORKLOADS["cross_720p"]
    x = synth.make_inputs(w)
    rows = synth.sample_rows(w.S, 256)
    check_fwd(x, rows=rows)


def test_cross_fwd_with_equal_lengths_is_the_self_attention_call():
    import torch
    import video_dit_full_b200 as wa
    x = inputs_for_cross(1, 390, 390, 2, seed=5)
    q, k, v = (to_device(x[n]) for n in "qkv")
    o1, l1 = wa.fwd(q, k, v)
    o2, l2 = wa.cross_fwd(q, k, v)
    wa.check_status()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def run_bwd(x):
    import video_dit_full_b200 as wa
    q, k, v, do = (to_device(x[n]) for n in ("q", "k", "v", "do"))
    o, lse = wa.cross_fwd(q, k, v)
    dq, dk, dv = wa.cross_bwd(q, k, v, o, do, lse)
    wa.check_status()
    return {"dq": bf16_to_f64(dq), "dk": bf16_to_f64(dk), "dv": bf16_to_f64(dv)}


def check_bwd(x, q_rows=None, k_rows=None, heads=None, by_head=False):
    got = run_bwd(x)
    if by_head:
        want = oracle_bwd_by_head(x, q_rows, k_rows, heads)
    else:
        want = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], q_rows=q_rows, k_rows=k_rows, heads=heads)
    sel = {"dq": q_rows, "dk": k_rows, "dv": k_rows}
    for name in ("dq", "dk", "dv"):
        g = got[name]
        if sel[name] is not None:
            g = g[:, sel[name]]
        if heads is not None:
            g = g[:, :, heads]
        if g.shape[1] == 0:
            continue
        assert np.all(np.isfinite(g))
        if not np.any(want[name]):            # Skv = 1: dQ = dK = 0 exactly
            assert np.abs(g).max() <= ZERO_GRAD_ABS, (name, np.abs(g).max())
            continue
        max_abs, rel = errors(g, want[name])
        print(f"{name}: max-abs {max_abs:.3e} rel-frob {rel:.3e}")
        assert rel <= GRAD_REL_FROB, (name, rel)
    return got


@pytest.mark.parametrize("B,Sq,Skv,H", [(1, 1, 1, 1), (1, 300, 77, 2), (2, 129, 512, 1), (1, 1000, 1, 2),
                                        (1, 520, 333, 3), (1, 256, 2048, 40)])
def test_cross_bwd_shapes_full(B, Sq, Skv, H):
    check_bwd(inputs_for_cross(B, Sq, Skv, H, seed=11 + Sq + Skv, with_do=True))


def test_cross_bwd_training_480p_text_sampled_rows():
    w = synth.WORKLOADS["cross_train_480p"]
    x = synth.make_inputs(w)
    q_rows = synth.sample_rows(w.S, 256, stream=synth.STREAM_QROWS)
    got = check_bwd(x, q_rows=q_rows, k_rows=[])                      # dQ rows, every head
    check_bwd(x, q_rows=[], k_rows=None, heads=list(range(w.H)), by_head=True)   # every key's dK, dV, every head
    # shifting every key by one vector leaves O unchanged, so sum_j dK_j = 0
    dk = got["dk"]
    assert np.linalg.norm(dk.sum(axis=1)) <= 1e-2 * np.linalg.norm(dk)
