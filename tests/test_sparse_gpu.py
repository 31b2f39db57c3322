"""Parity of the block-sparse forward (wan_attn_fwd_block_sparse, through the C ABI) with the oracle
(oracle/block_sparse.py): the bf16 forward's bars (O max-abs 1e-2 and rel-Frobenius 5e-3, LSE
1e-3) on the rows that attend something; rows that attend nothing must be exactly O = 0,
LSE = -inf.  An all-ones mask must agree with wan_attn_fwd to rounding (the two kernels mix
their exponentials differently and rescale at different points).  The per-tile key-block lists
the call builds in its workspace must equal, entry for entry, the lists built on the host from the
mask (integer work: bit-exact)."""
import numpy as np
import pytest

import synth
from gpu_util import bf16_to_f64, errors, inputs_for_cross, to_device
from oracle import block_sparse as bs

pytestmark = pytest.mark.gpu

O_MAX_ABS, O_REL_FROB, LSE_MAX_ABS = 1e-2, 5e-3, 1e-3


def run(x, mask):
    import torch
    import video_dit_full_b200 as wa
    q, k, v = (to_device(x[n]) for n in "qkv")
    m = torch.from_numpy(np.ascontiguousarray(mask)).cuda()
    o, lse = wa.fwd_block_sparse(q, k, v, m)
    wa.check_status()
    return o, lse


def check(x, mask, rows=None, heads=None):
    o, lse = run(x, mask)
    want_o, want_lse = bs.attn_fwd_block_sparse(x["q"], x["k"], x["v"], mask, rows=rows, heads=heads)
    got_o, got_lse = bf16_to_f64(o), lse.cpu().numpy().astype(np.float64)
    if rows is not None:
        got_o, got_lse = got_o[:, rows], got_lse[:, :, rows]
    if heads is not None:
        got_o, got_lse = got_o[:, :, heads], got_lse[:, heads]
    empty = np.isneginf(want_lse)                                    # [B, H, R]
    assert np.all(np.isneginf(got_lse[empty]))
    assert np.all(got_o.transpose(0, 2, 1, 3)[empty] == 0)
    live = ~empty
    go, wo = got_o.transpose(0, 2, 1, 3)[live], want_o.transpose(0, 2, 1, 3)[live]
    if go.size:
        max_abs, rel = errors(go, wo)
        lse_err = float(np.abs(got_lse[live] - want_lse[live]).max())
        print(f"O max-abs {max_abs:.3e} rel-frob {rel:.3e}  LSE max-abs {lse_err:.3e}  empty rows {empty.sum()}")
        assert max_abs <= O_MAX_ABS and rel <= O_REL_FROB, (max_abs, rel)
        assert lse_err <= LSE_MAX_ABS, lse_err


def test_all_ones_mask_matches_the_dense_call():
    import video_dit_full_b200 as wa
    x = inputs_for_cross(2, 1000, 1000, 3, seed=21)
    mask = np.ones((2, 3, bs.blocks(1000), bs.blocks(1000)), dtype=np.uint8)
    check(x, mask)
    o, lse = run(x, mask)
    q, k, v = (to_device(x[n]) for n in "qkv")
    od, ld = wa.fwd(q, k, v)
    wa.check_status()
    # each call is within the forward's bars of the exact result (bf16 output rounding, ~2.3e-3
    # rel-Frobenius apiece), so the two are within the sum of those bars of each other
    max_abs, rel = errors(bf16_to_f64(o), bf16_to_f64(od))
    assert rel <= 2 * O_REL_FROB and max_abs <= 2 * O_MAX_ABS, (rel, max_abs)
    assert float((lse - ld).abs().max()) <= 2 * LSE_MAX_ABS


# (1, 1), (129, 64): one key block, a single step; (200, 100): two steps, the next-to-last
# product's barrier at step 0; (300, 130): three steps, the last one short
@pytest.mark.parametrize("Sq,Skv,keep", [(1000, 1000, 0.5), (1000, 1000, 0.125), (300, 777, 0.25),
                                         (4100, 4100, 0.125), (65, 64, 1.0), (1, 1, 1.0), (129, 64, 1.0),
                                         (200, 100, 1.0), (300, 130, 1.0)])
def test_random_masks(Sq, Skv, keep):
    B, H = 1, 2
    x = inputs_for_cross(B, Sq, Skv, H, seed=Sq + Skv)
    mask = synth.block_mask(B, H, bs.blocks(Sq), bs.blocks(Skv), keep, seed=Sq)
    check(x, mask)


def test_rows_and_ctas_that_attend_nothing():
    B, H, S = 1, 2, 1300
    x = inputs_for_cross(B, S, S, H, seed=4)
    mask = synth.block_mask(B, H, bs.blocks(S), bs.blocks(S), 0.3, seed=4)
    mask[0, 0, 1] = 0                     # one query block of head 0
    mask[0, 1, 4:8] = 0                   # every query block of CTA 1 (tokens 256-511) of head 1
    mask[0, 1, 20] = 0                    # the short last block
    check(x, mask)


def test_block_diagonal_mask():
    B, H, S = 1, 2, 777
    x = inputs_for_cross(B, S, S, H, seed=5)
    nb = bs.blocks(S)
    mask = np.zeros((B, H, nb, nb), dtype=np.uint8)
    for i in range(nb):
        mask[:, :, i, i] = 1
    check(x, mask)


def test_720p_at_one_eighth_density_sampled_rows():
    w = synth.WORKLOADS["wan14b_720p"]
    x = synth.make_inputs(w)
    nb = bs.blocks(w.S)
    mask = synth.block_mask(w.B, w.H, nb, nb, 0.125, seed=0)
    check(x, mask, rows=synth.sample_rows(w.S, 256))


def test_tiles_that_need_one_half_or_start_late():
    # Each CTA's tiles (query blocks 0-1 and 2-3 of its four) get their own MMAs:
    # head 0: tile 0 attends even key blocks, tile 1 odd ones, so every step's two blocks split
    #         between the tiles and each tile runs one 64-key half of it;
    # head 1: tile 1 attends key blocks 0-2 only, tile 0 blocks 12.. only, the short last one
    #         included, so tile 0 has no product for its first step and later steps start it.
    B, H, S = 1, 2, 1500
    x = inputs_for_cross(B, S, S, H, seed=12)
    nb = bs.blocks(S)
    mask = np.zeros((B, H, nb, nb), dtype=np.uint8)
    for qb in range(nb):
        tile = (qb % 4) // 2
        mask[0, 0, qb, tile::2] = 1
        if tile == 0:
            mask[0, 1, qb, 12:] = 1
        else:
            mask[0, 1, qb, :3] = 1
    check(x, mask)


def tile_lists_from_mask(mask):
    """Each 128-row Q tile's ascending union of the key blocks its two query blocks attend, one
    int32 entry per block: the block index, bit 30 set if the first query block attends it, bit 31
    if the second does; and the union's length.  Built from the mask alone."""
    B, H, nqb, nkb = mask.shape
    ntiles = (nqb + 1) // 2
    lists = np.zeros((B, H, ntiles, nkb), dtype=np.uint32)
    counts = np.zeros((B, H, ntiles), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for t in range(ntiles):
                r0 = mask[b, h, 2 * t] != 0
                r1 = mask[b, h, 2 * t + 1] != 0 if 2 * t + 1 < nqb else np.zeros(nkb, dtype=bool)
                kb = np.nonzero(r0 | r1)[0]
                entries = kb.astype(np.uint32) | (r0[kb].astype(np.uint32) << 30) | (r1[kb].astype(np.uint32) << 31)
                lists[b, h, t, :kb.size] = entries
                counts[b, h, t] = kb.size
    return lists, counts


@pytest.mark.parametrize("Sq,Skv,keep", [(1300, 900, 0.3), (65, 64, 1.0), (4100, 333, 0.125)])
def test_tile_lists_in_the_workspace_are_exact(Sq, Skv, keep):
    # Integer work: the per-tile lists the call builds in its workspace must equal the ones built
    # from the mask on the host, entry for entry (the workspace is int32 lists [B, H, ntiles, nkb]
    # then, 256-byte aligned, the lengths [B, H, ntiles]; list entries past a length are unused).
    import torch
    import video_dit_full_b200 as wa
    B, H = 2, 3
    x = inputs_for_cross(B, Sq, Skv, H, seed=Sq)
    mask = synth.block_mask(B, H, bs.blocks(Sq), bs.blocks(Skv), keep, seed=Skv)
    q, k, v = (to_device(x[n]) for n in "qkv")
    ws = torch.zeros(wa.block_sparse_workspace_size(B, Sq, Skv, H), dtype=torch.uint8, device="cuda")
    wa.fwd_block_sparse(q, k, v, torch.from_numpy(mask).cuda(), workspace=ws)
    wa.check_status()
    want_lists, want_counts = tile_lists_from_mask(mask)
    ntiles, nkb = want_lists.shape[2], want_lists.shape[3]
    list_bytes = B * H * ntiles * nkb * 4
    raw = ws.cpu().numpy()
    got_lists = raw[:list_bytes].view(np.uint32).reshape(B, H, ntiles, nkb)
    off = (list_bytes + 255) // 256 * 256
    got_counts = raw[off:off + B * H * ntiles * 4].view(np.int32).reshape(B, H, ntiles)
    assert np.array_equal(got_counts, want_counts)
    for b in range(B):
        for h in range(H):
            for t in range(ntiles):
                n = want_counts[b, h, t]
                assert np.array_equal(got_lists[b, h, t, :n], want_lists[b, h, t, :n]), (b, h, t)
