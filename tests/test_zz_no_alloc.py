"""wan_attn_bwd_noalloc: the backward for callers that cannot allocate device memory.

Such callers (a plugin whose host owns all device memory, a server that bans
cudaMalloc after start-up) pass only inputs and outputs; the workspace is a
fixed array inside the library.  These tests call it through the C ABI and
compare it with wan_attn_bwd given a caller workspace, on two calls in a row.
The tolerance is the backward's: relative Frobenius error <= 2e-2 (dQ is
summed across key tiles by asynchronous fp32 reduce-adds in no fixed order, so
its low bits may differ between runs; dK and dV are deterministic and must
match exactly).  One case sits just under the array's limit, so the last bytes
of the array (where D_i lives) and the dQ accumulator spanning nearly all of it
are exercised.
"""
import ctypes

import numpy as np
import pytest

from gpu_util import inputs_for, to_device

REL_FROB = 2e-2
LIMIT = 32 << 20          # WAN_ATTN_NOALLOC_WORKSPACE_BYTES


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_limit_is_rejected_on_the_host(built):
    from video_dit_full_b200 import wan_attn
    lib = wan_attn.lib()
    fake = [ctypes.c_void_p(0x100000 + i * 0x10000000) for i in range(9)]
    rows_max = 65027
    assert lib.wan_attn_bwd_workspace_size(1, rows_max, 1, 128) <= LIMIT
    assert lib.wan_attn_bwd_workspace_size(1, rows_max + 1, 1, 128) > LIMIT
    # too large for the library's array: rejected before anything is enqueued
    assert lib.wan_attn_bwd_noalloc(*fake, 1, rows_max + 1, 1, 128, None) == 5      # WAN_ATTN_ERR_WORKSPACE
    assert lib.wan_attn_bwd_noalloc(*fake, 2, 4096, 24, 128, None) == 5
    assert lib.wan_attn_bwd_noalloc(*fake, 1, 128, 1, 64, None) == 2                # head dim: unsupported
    assert lib.wan_attn_bwd_noalloc(None, *fake[1:], 1, 128, 1, 128, None) == 1     # null input


@pytest.mark.gpu
@pytest.mark.parametrize("B,S,H", [(1, 1000, 3), (1, 2048, 31)])
def test_noalloc_matches_workspace_backward_twice(B, S, H):
    import torch
    import video_dit_full_b200 as wa
    from video_dit_full_b200 import wan_attn
    lib = wan_attn.lib()
    D = 128
    assert lib.wan_attn_bwd_workspace_size(B, S, H, D) <= LIMIT
    x = inputs_for(B, S, H, seed=21 + H, with_do=True)
    q, k, v, do = (to_device(x[n]) for n in ("q", "k", "v", "do"))
    o, lse = wa.fwd(q, k, v)
    ref_dq, ref_dk, ref_dv = wa.bwd(q, k, v, o, do, lse)
    wa.check_status()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
        st = lib.wan_attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse),
                                      _ptr(dq), _ptr(dk), _ptr(dv), B, S, H, D, stream)
        assert st == 0, st
        assert wa.sync_status() == 0
        for name, got, ref in (("dq", dq, ref_dq), ("dk", dk, ref_dk), ("dv", dv, ref_dv)):
            g = got.float().cpu().numpy().astype(np.float64)
            r = ref.float().cpu().numpy().astype(np.float64)
            assert np.all(np.isfinite(g)), (call, name)
            rel = np.linalg.norm(g - r) / np.linalg.norm(r)
            assert rel <= REL_FROB, (call, name, rel)
        assert torch.equal(dk, ref_dk) and torch.equal(dv, ref_dv)
