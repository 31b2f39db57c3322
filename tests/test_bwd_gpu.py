"""Parity of the bf16 backward (wan_attn_bwd through the C ABI) with the fp64 oracle.

Bar (the training workload's stated tolerance): relative Frobenius error
<= 2e-2 for each of dQ, dK and dV.  The GPU backward consumes the GPU
forward's own O and LSE, as a training step does; the oracle differentiates
its own fp64 forward.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import bf16_to_f64, errors, inputs_for, oracle_bwd_by_head, to_device

pytestmark = pytest.mark.gpu

REL_FROB = 2e-2


def run_bwd(x):
    import video_dit_full_b200 as wa
    q, k, v, do = (to_device(x[n]) for n in ("q", "k", "v", "do"))
    o, lse = wa.fwd(q, k, v)
    dq, dk, dv = wa.bwd(q, k, v, o, do, lse)
    wa.check_status()
    return dq, dk, dv


def check(x, q_rows=None, k_rows=None, heads=None, by_head=False):
    dq, dk, dv = run_bwd(x)
    if by_head:
        want = oracle_bwd_by_head(x, q_rows, k_rows, heads)
    else:
        want = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], q_rows=q_rows, k_rows=k_rows, heads=heads)
    got = {"dq": bf16_to_f64(dq), "dk": bf16_to_f64(dk), "dv": bf16_to_f64(dv)}
    sel = {"dq": q_rows, "dk": k_rows, "dv": k_rows}
    out = {}
    for name in ("dq", "dk", "dv"):
        g = got[name]
        if sel[name] is not None:
            g = g[:, sel[name]]
        if heads is not None:
            g = g[:, :, heads]
        if g.shape[1] == 0:
            continue
        assert np.all(np.isfinite(g))
        if not np.any(want[name]):            # e.g. S = 1: dQ = dK = 0 exactly
            assert np.abs(g).max() <= 1e-6, (name, np.abs(g).max())
            continue
        max_abs, rel = errors(g, want[name])
        out[name] = rel
        print(f"{name}: max-abs {max_abs:.3e} rel-frob {rel:.3e}")
        assert rel <= REL_FROB, (name, rel)
    return got, out


@pytest.mark.parametrize("B,S,H", [(1, 1, 1), (1, 2, 2), (2, 65, 1), (1, 128, 2), (1, 129, 1), (2, 255, 2),
                                   (1, 300, 3), (1, 1000, 2)])
def test_bwd_ragged_shapes_full(B, S, H):
    check(inputs_for(B, S, H, seed=100 + S, with_do=True))


def test_bwd_oracle_sized_shape_full():
    check(inputs_for(1, 1280, 12, seed=0, with_do=True))


def test_bwd_peaky_scores():
    check(inputs_for(1, 700, 2, seed=7, with_do=True, q_mul=4.0))


def test_bwd_training_480p_sampled_rows():
    w = synth.WORKLOADS["train_480p_fwd_bwd"]
    x = synth.make_inputs(w)
    q_rows = synth.sample_rows(w.S, 256, stream=synth.STREAM_QROWS)
    k_rows = synth.sample_rows(w.S, 256, stream=synth.STREAM_KROWS)
    got, _ = check(x, q_rows=q_rows, k_rows=[])                  # dQ rows, every head
    # dK, dV of the 256 key rows on every head: each head needs the fp64 LSE and D_i of all
    # 32760 query rows (a full forward per head), computed one head per host thread
    check(x, q_rows=[], k_rows=k_rows, heads=list(range(w.H)), by_head=True)
    # any size: shifting every key by one vector leaves O unchanged, so sum_j dK_j = 0
    dk = got["dk"]
    col = dk.sum(axis=1)
    assert np.linalg.norm(col) <= 1e-2 * np.linalg.norm(dk)
