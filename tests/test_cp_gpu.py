"""The context-parallel kernels (wan_attn_cp_merge, wan_attn_cp_accumulate, wan_attn_cp_layout)
and the Ring / Ulysses schedules on one GPU.  G ranks are G threads exchanging tensors by
host-synchronised copies (tests/cp_helpers.ThreadComm): every compute step is the CUDA
library's, and no kernel waits on another.

Bars: the merged O as the bf16 forward (max-abs 1e-2, rel-Frobenius 5e-3, LSE 1e-3); the
schedules' gradients as the backward (rel-Frobenius 2e-2); accumulate and layout bit-exact.
"""
import numpy as np
import pytest

import oracle
import synth
from cp_helpers import run_threads
from gpu_util import bf16_to_f64, errors, inputs_for_cross, to_device

pytestmark = pytest.mark.gpu

O_MAX_ABS, O_REL_FROB, LSE_MAX_ABS, GRAD_REL_FROB = 1e-2, 5e-3, 1e-3, 2e-2


def check_o(o, lse, want_o, want_lse):
    got_o = bf16_to_f64(o)
    got_lse = lse.cpu().numpy().astype(np.float64)
    max_abs, rel = errors(got_o, want_o)
    lse_err = float(np.abs(got_lse - want_lse).max())
    print(f"O max-abs {max_abs:.3e} rel-frob {rel:.3e}  LSE max-abs {lse_err:.3e}")
    assert max_abs <= O_MAX_ABS and rel <= O_REL_FROB, (max_abs, rel)
    assert lse_err <= LSE_MAX_ABS, lse_err


def check_grads(got, want):
    for name, g in zip(("dq", "dk", "dv"), got):
        max_abs, rel = errors(bf16_to_f64(g), want[name])
        print(f"{name}: max-abs {max_abs:.3e} rel-frob {rel:.3e}")
        assert rel <= GRAD_REL_FROB, (name, rel)


@pytest.mark.parametrize("chunks", [[1000], [300, 129, 571], [1, 999]])
def test_merge_of_key_blocks_is_the_whole_softmax(chunks):
    import torch
    import video_dit_full_b200 as wa
    Sq, H = 600, 3
    x = inputs_for_cross(1, Sq, sum(chunks), H, seed=len(chunks))
    q, k, v = (to_device(x[n]) for n in "qkv")
    o_acc = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    lse = torch.empty((1, H, Sq), dtype=torch.float32, device="cuda")
    o = torch.empty_like(q)
    j0 = 0
    for i, n in enumerate(chunks):
        o_t, lse_t = wa.cross_fwd(q, k[:, j0:j0 + n].contiguous(), v[:, j0:j0 + n].contiguous())
        wa.cp_merge(o_acc, lse, o_t, lse_t, i == 0, o if i + 1 == len(chunks) else None)
        j0 += n
    wa.check_status()
    want_o, want_lse = oracle.attn_fwd(x["q"], x["k"], x["v"])
    check_o(o, lse, want_o, want_lse)
    # the fp32 running O is the bf16 output before rounding
    assert torch.equal(o_acc.to(torch.bfloat16), o)


def test_accumulate_is_the_fp32_sum_in_order():
    import torch
    import video_dit_full_b200 as wa
    n = 3 * 8 * 1001
    parts = [synth.make_tensor((n,), 3, s) for s in range(3)]
    acc = torch.empty(n, dtype=torch.float32, device="cuda")
    out = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    for i, p in enumerate(parts):
        wa.cp_accumulate(acc, to_device(p), i == 0, out if i == 2 else None)
    wa.check_status()
    f = [synth.bf16_bits_to_f32(p) for p in parts]
    want = (f[0] + f[1]) + f[2]                         # fp32, the same order
    np.testing.assert_array_equal(acc.cpu().numpy(), want)
    want_bits = synth.f64_to_bf16_bits(want.astype(np.float64))   # exact: fp32 -> fp64 -> bf16 RNE
    np.testing.assert_array_equal(out.cpu().view(torch.int16).numpy().view(np.uint16), want_bits)


@pytest.mark.parametrize("B,S_loc,G,Hg", [(1, 5, 4, 2), (2, 3, 3, 1), (3, 130, 2, 5)])
def test_layout_permutations(B, S_loc, G, Hg):
    import torch
    import video_dit_full_b200 as wa
    D = 128
    src = to_device(synth.make_tensor((B * S_loc * G * Hg * D,), 9, 0))
    dst = torch.empty_like(src)
    want = {
        wa.CP_SEQ_TO_SEND: src.view(B, S_loc, G, Hg, D).permute(2, 0, 1, 3, 4),
        wa.CP_RECV_TO_HEADS: src.view(G, B, S_loc, Hg, D).permute(1, 0, 2, 3, 4),
        wa.CP_HEADS_TO_SEND: src.view(B, G, S_loc, Hg, D).permute(1, 0, 2, 3, 4),
        wa.CP_RECV_TO_SEQ: src.view(G, B, S_loc, Hg, D).permute(1, 2, 0, 3, 4),
    }
    for which, y in want.items():
        wa.cp_layout(dst, src, B, S_loc, G, Hg, which)
        wa.check_status()
        assert torch.equal(dst, y.contiguous().view(-1)), which


def _shards(x, G, S_loc, r):
    return [to_device(np.ascontiguousarray(x[n][:, r * S_loc:(r + 1) * S_loc])) for n in ("q", "k", "v", "do")]


@pytest.mark.parametrize("G,B,S_loc,H", [(3, 1, 200, 4), (2, 2, 256, 2), (4, 1, 97, 3)])
def test_ring_schedule_on_virtual_ranks(G, B, S_loc, H):
    from video_dit_full_b200 import context_parallel as cp
    x = inputs_for_cross(B, G * S_loc, G * S_loc, H, seed=G * S_loc, with_do=True)

    def rank(r, comm):
        q, k, v, do = _shards(x, G, S_loc, r)
        o, lse = cp.ring_attn_fwd(q, k, v, comm)
        grads = cp.ring_attn_bwd(q, k, v, o, do, lse, comm)
        return o, lse, grads

    res = run_threads(G, rank)
    import torch
    o = torch.cat([r[0] for r in res], dim=1)
    lse = torch.cat([r[1] for r in res], dim=2)
    want_o, want_lse = oracle.attn_fwd(x["q"], x["k"], x["v"])
    check_o(o, lse, want_o, want_lse)
    grads = [torch.cat([r[2][i] for r in res], dim=1) for i in range(3)]
    check_grads(grads, oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"]))


@pytest.mark.parametrize("G,B,S_loc,H", [(2, 2, 200, 4), (4, 1, 128, 8), (3, 1, 65, 3)])
def test_ulysses_schedule_on_virtual_ranks(G, B, S_loc, H):
    import torch
    from video_dit_full_b200 import context_parallel as cp
    x = inputs_for_cross(B, G * S_loc, G * S_loc, H, seed=7 + G * S_loc, with_do=True)

    def rank(r, comm):
        q, k, v, do = _shards(x, G, S_loc, r)
        o, ctx = cp.ulysses_attn_fwd(q, k, v, comm)
        return o, cp.ulysses_attn_bwd(do, ctx, comm)

    res = run_threads(G, rank)
    o = torch.cat([r[0] for r in res], dim=1)
    want_o, want_lse = oracle.attn_fwd(x["q"], x["k"], x["v"])
    max_abs, rel = errors(bf16_to_f64(o), want_o)
    assert max_abs <= O_MAX_ABS and rel <= O_REL_FROB, (max_abs, rel)
    grads = [torch.cat([r[1][i] for r in res], dim=1) for i in range(3)]
    check_grads(grads, oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"]))


def test_single_rank_schedules_are_the_plain_calls():
    import torch
    import video_dit_full_b200 as wa
    from video_dit_full_b200 import context_parallel as cp
    x = inputs_for_cross(1, 300, 300, 2, seed=3, with_do=True)
    q, k, v, do = (to_device(x[n]) for n in ("q", "k", "v", "do"))
    o, lse = wa.fwd(q, k, v)
    o_r, lse_r = cp.ring_attn_fwd(q, k, v)
    o_u, _ = cp.ulysses_attn_fwd(q, k, v)
    wa.check_status()
    assert torch.equal(o_u, o)
    assert torch.equal(o_r, o) and torch.allclose(lse_r, lse, rtol=0, atol=1e-6)
