"""The C-ABI library loads on a machine without a GPU, exports every entry point
the header declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "wan_attn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(wan_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("wan_attn_fwd", "wan_attn_sync_status", "wan_attn_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(built):
    out = subprocess.check_output(["nm", "-D", "--defined-only", built], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    # nothing else of ours leaks out of the shared object
    ours = sorted(n for n in exported if n.startswith("wan"))
    assert ours == declared_functions()


def test_binding_covers_every_symbol(built):
    from video_dit_full_b200 import wan_attn
    assert sorted(n for n, _, _ in wan_attn.SIGNATURES) == declared_functions()
    lib = wan_attn.lib()
    for name in declared_functions():
        assert getattr(lib, name)


def test_host_side_validation_without_gpu(built):
    from video_dit_full_b200 import wan_attn
    lib = wan_attn.lib()
    p = ctypes.c_void_p(0x10000)      # aligned fake addresses: never dereferenced on these paths
    p2, p3, p4, p5 = (ctypes.c_void_p(0x10000 + i * 0x1000000) for i in range(1, 5))
    INVALID, UNSUPPORTED = 1, 2
    assert lib.wan_attn_fwd(None, p2, p3, p4, p5, 1, 128, 1, 128, None) == INVALID
    assert lib.wan_attn_fwd(p, p2, p3, p4, None, 1, 128, 1, 128, None) == INVALID
    assert lib.wan_attn_fwd(p, p2, p3, p4, p5, 0, 128, 1, 128, None) == INVALID
    assert lib.wan_attn_fwd(p, p2, p3, p4, p5, 1, -5, 1, 128, None) == INVALID
    assert lib.wan_attn_fwd(p, p2, p3, p4, p5, 1, 128, 1, 64, None) == UNSUPPORTED
    odd = ctypes.c_void_p(0x10008)
    assert lib.wan_attn_fwd(odd, p2, p3, p4, p5, 1, 128, 1, 128, None) == INVALID
    # output overlapping an input
    assert lib.wan_attn_fwd(p, p2, p3, p, p5, 1, 128, 1, 128, None) == INVALID
    # lse overlapping o
    assert lib.wan_attn_fwd(p, p2, p3, p4, ctypes.c_void_p(0x10000 + 3 * 0x1000000 + 64), 1, 128, 1, 128,
                            None) == INVALID
    assert lib.wan_attn_status_string(4) == b"a kernel wait ran out of time"
    old = lib.wan_attn_set_wait_budget_ns(5)
    assert lib.wan_attn_set_wait_budget_ns(old) == 1000


def test_bwd_host_side_validation_without_gpu(built):
    from video_dit_full_b200 import wan_attn
    lib = wan_attn.lib()
    ptr = [ctypes.c_void_p(0x100000 + i * 0x1000000) for i in range(11)]
    q, k, v, o, do, lse, dq, dk, dv, ws = ptr[:10]
    need = lib.wan_attn_bwd_workspace_size(1, 128, 2, 128)
    assert need == 128 * 2 * 128 * 4 + 256 * 4
    assert lib.wan_attn_bwd_workspace_size(1, 128, 2, 64) == 0
    args = lambda **kw: [kw.get(n, d) for n, d in zip(
        ["q", "k", "v", "o", "do", "lse", "dq", "dk", "dv", "B", "S", "H", "D", "ws", "wsb", "st"],
        [q, k, v, o, do, lse, dq, dk, dv, 1, 128, 2, 128, ws, need, None])]
    INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 5
    assert lib.wan_attn_bwd(*args(do=None)) == INVALID
    assert lib.wan_attn_bwd(*args(D=96)) == UNSUPPORTED
    assert lib.wan_attn_bwd(*args(ws=None)) == WORKSPACE
    assert lib.wan_attn_bwd(*args(wsb=need - 1)) == WORKSPACE
    assert lib.wan_attn_bwd(*args(ws=ctypes.c_void_p(0x100000 + 9 * 0x1000000 + 16))) == WORKSPACE
    assert lib.wan_attn_bwd(*args(dq=q)) == INVALID                 # output aliases an input
    assert lib.wan_attn_bwd(*args(dk=dv)) == INVALID                # two outputs alias


def test_q8_host_side_validation_without_gpu(built):
    from video_dit_full_b200 import wan_attn
    lib = wan_attn.lib()
    q, k, v, o, lse, ws = (ctypes.c_void_p(0x100000 + i * 0x10000000) for i in range(6))
    need = lib.wan_attn_fwd_q8_workspace_size(1, 130, 2, 128)
    assert need == 3 * 33280 + 3 * 256      # 3 x align256(130*2*128) + 3 x align256(2*3*4)
    assert lib.wan_attn_fwd_q8_workspace_size(1, 130, 2, 100) == 0
    assert lib.wan_attn_fwd_q8(q, k, v, o, lse, 1, 130, 2, 128, None, need, None) == 5
    assert lib.wan_attn_fwd_q8(q, k, v, o, lse, 1, 130, 2, 128, ws, need - 1, None) == 5
    assert lib.wan_attn_fwd_q8(q, k, v, q, lse, 1, 130, 2, 128, ws, need, None) == 1
    assert lib.wan_attn_fwd_q8(q, k, v, o, lse, 1, 130, 2, 120, ws, need, None) == 2


def test_cross_host_side_validation_without_gpu(built):
    from video_dit_full_b200 import wan_attn
    lib = wan_attn.lib()
    INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 5
    q, k, v, o, lse = (ctypes.c_void_p(0x100000 + i * 0x10000000) for i in range(5))
    kv_bytes = 1 * 77 * 2 * 128 * 2
    # Skv is validated on its own, and K, V are sized by it
    assert lib.wan_attn_cross_fwd(q, k, v, o, lse, 1, 300, 0, 2, 128, None) == INVALID
    assert lib.wan_attn_cross_fwd(q, k, v, o, lse, 1, 300, 77, 2, 64, None) == UNSUPPORTED
    assert lib.wan_attn_cross_fwd(q, k, v, ctypes.c_void_p(k.value + kv_bytes - 256), lse, 1, 300, 77, 2, 128,
                                  None) == INVALID     # o starts inside k
    # workspace: dQ acc [Sq] + D_i [Sq] + dK, dV accumulators [Skv]
    need = lib.wan_attn_cross_bwd_workspace_size(1, 300, 77, 2, 128)
    a = lambda x: (x + 255) // 256 * 256
    assert need == a(300 * 2 * 128 * 4) + a(2 * 300 * 4) + 2 * a(77 * 2 * 128 * 4)
    assert lib.wan_attn_cross_bwd_workspace_size(1, 300, 0, 2, 128) == 0
    ptr = [ctypes.c_void_p(0x100000 + i * 0x1000000) for i in range(10)]
    q, k, v, o, do, lse, dq, dk, dv, ws = ptr
    args = lambda **kw: [kw.get(n, d) for n, d in zip(
        ["q", "k", "v", "o", "do", "lse", "dq", "dk", "dv", "B", "Sq", "Skv", "H", "D", "ws", "wsb", "st"],
        [q, k, v, o, do, lse, dq, dk, dv, 1, 300, 77, 2, 128, ws, need, None])]
    assert lib.wan_attn_cross_bwd(*args(ws=None)) == WORKSPACE
    assert lib.wan_attn_cross_bwd(*args(wsb=need - 1)) == WORKSPACE
    assert lib.wan_attn_cross_bwd(*args(Skv=-1)) == INVALID
    assert lib.wan_attn_cross_bwd(*args(D=256)) == UNSUPPORTED
    assert lib.wan_attn_cross_bwd(*args(dk=v)) == INVALID                 # output aliases an input
    assert lib.wan_attn_cross_bwd(*args(dv=ctypes.c_void_p(dk.value + 64))) == INVALID   # outputs overlap


def test_sparse_fp8_cp_host_side_validation_without_gpu(built):
    from video_dit_full_b200 import wan_attn
    lib = wan_attn.lib()
    INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 5
    P = [ctypes.c_void_p(0x100000 + i * 0x10000000) for i in range(8)]
    q, k, v, o, lse, mask, ws, z = P
    # block-sparse: lists int32 [B, H, ceil(Sq/128), ceil(Skv/64)] + lengths, each 256-byte aligned
    need = lib.wan_attn_fwd_block_sparse_workspace_size(1, 300, 700, 2, 128)
    a = lambda x: (x + 255) // 256 * 256
    assert need == a(2 * 3 * 11 * 4) + a(2 * 3 * 4)
    assert lib.wan_attn_fwd_block_sparse_workspace_size(1, 300, 700, 2, 96) == 0
    args = [q, k, v, o, lse, mask, 1, 300, 700, 2, 128, ws, need, None]
    assert lib.wan_attn_fwd_block_sparse(*args[:5], None, *args[6:]) == INVALID          # no mask
    assert lib.wan_attn_fwd_block_sparse(*args[:10], 64, *args[11:]) == UNSUPPORTED
    assert lib.wan_attn_fwd_block_sparse(*args[:12], need - 4, None) == WORKSPACE
    assert lib.wan_attn_fwd_block_sparse(*args[:11], None, need, None) == WORKSPACE
    assert lib.wan_attn_fwd_block_sparse(q, k, v, q, *args[4:]) == INVALID               # o aliases q
    # FP8: K a multiple of 16, N of 8, outputs overlap no input
    assert lib.wan_fp8_quantize_rows(q, k, v, 10, 24, None) == INVALID
    assert lib.wan_fp8_quantize_rows(q, q, v, 10, 32, None) == INVALID
    assert lib.wan_fp8_quantize_tensor(q, k, ctypes.c_void_p(v.value + 4), 8, 32, None) == INVALID  # scale2 8-aligned
    assert lib.wan_fp8_gemm(q, k, v, o, lse, 100, 20, 32, None) == INVALID               # N % 8
    assert lib.wan_fp8_gemm(q, k, v, o, q, 100, 24, 32, None) == INVALID                 # y aliases the codes
    assert lib.wan_fp8_gemm(None, k, v, o, lse, 100, 24, 32, None) == INVALID
    # context parallelism
    assert lib.wan_attn_cp_accumulate(q, k, None, 12, 1, None) == INVALID                # n % 8
    assert lib.wan_attn_cp_accumulate(q, ctypes.c_void_p(q.value + 16), None, 64, 0, None) == INVALID
    assert lib.wan_attn_cp_layout(q, k, 1, 5, 2, 2, 128, 4, None) == INVALID             # no such order
    assert lib.wan_attn_cp_layout(q, k, 1, 5, 2, 2, 64, 0, None) == UNSUPPORTED
    assert lib.wan_attn_cp_merge(q, k, q, o, None, 1, 10, 2, 128, 0, None) == INVALID    # o_part aliases o_acc
    assert lib.wan_attn_cp_merge(q, k, v, None, None, 1, 10, 2, 128, 0, None) == INVALID  # no lse_part
