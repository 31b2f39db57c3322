"""Thin ctypes binding of ``libwan_attn.so`` (the C ABI in ``include/wan_attn.h``).

Argument marshalling only: torch tensors are checked for dtype, device, shape
and contiguity, and their device pointers and the current CUDA stream are
passed to the library, which runs every step of the computation in its own
kernels.  There is no fallback: if the library is missing or a call fails, an
exception is raised.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libwan_attn.so")

STATUS = {0: "WAN_ATTN_OK", 1: "WAN_ATTN_ERR_INVALID_ARG", 2: "WAN_ATTN_ERR_UNSUPPORTED",
          3: "WAN_ATTN_ERR_CUDA", 4: "WAN_ATTN_ERR_TIMEOUT", 5: "WAN_ATTN_ERR_WORKSPACE"}

# (name, restype, argtypes) of every entry point the header declares
_P, _I, _Z, _U64, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64, ctypes.c_void_p
SIGNATURES = [
    ("wan_attn_fwd", _I, [_P, _P, _P, _P, _F, _I, _I, _I, _I, _P]),
    ("wan_attn_bwd_workspace_size", _Z, [_I, _I, _I, _I]),
    ("wan_attn_bwd", _I, [_P, _P, _P, _P, _P, _F, _P, _P, _P, _I, _I, _I, _I, _P, _Z, _P]),
    ("wan_attn_cross_fwd", _I, [_P, _P, _P, _P, _F, _I, _I, _I, _I, _I, _P]),
    ("wan_attn_cross_bwd_workspace_size", _Z, [_I, _I, _I, _I, _I]),
    ("wan_attn_cross_bwd", _I, [_P, _P, _P, _P, _P, _F, _P, _P, _P, _I, _I, _I, _I, _I, _P, _Z, _P]),
    ("wan_attn_cp_merge", _I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    ("wan_attn_cp_accumulate", _I, [_P, _P, _P, _Z, _I, _P]),
    ("wan_attn_cp_layout", _I, [_P, _P, _I, _I, _I, _I, _I, _I, _P]),
    ("wan_attn_fwd_block_sparse_workspace_size", _Z, [_I, _I, _I, _I, _I]),
    ("wan_attn_fwd_block_sparse", _I, [_P, _P, _P, _P, _F, _P, _I, _I, _I, _I, _I, _P, _Z, _P]),
    ("wan_fp8_quantize_rows", _I, [_P, _P, _P, _I, _I, _P]),
    ("wan_fp8_quantize_tensor", _I, [_P, _P, _P, _I, _I, _P]),
    ("wan_fp8_gemm", _I, [_P, _P, _P, _P, _P, _I, _I, _I, _P]),
    ("wan_attn_fwd_q8_workspace_size", _Z, [_I, _I, _I, _I]),
    ("wan_attn_fwd_q8", _I, [_P, _P, _P, _P, _F, _I, _I, _I, _I, _P, _Z, _P]),
    ("wan_attn_bwd_noalloc", _I, [_P, _P, _P, _P, _P, _F, _P, _P, _P, _I, _I, _I, _I, _P]),
    ("wan_attn_sync_status", _I, [_P]),
    ("wan_attn_status_string", ctypes.c_char_p, [_I]),
    ("wan_attn_set_wait_budget_ns", _U64, [_U64]),
    ("wan_attn_selftest_wait_timeout", _I, [_U64, _P]),
]


class WanAttnError(RuntimeError):
    def __init__(self, call: str, status: int):
        self.status = status
        super().__init__(f"{call} failed: {STATUS.get(status, status)}")


_lib = None


def lib():
    """Load the library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m video_dit_full_b200.build` "
                               "(there is no fallback implementation)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _check(call: str, status: int):
    if status != 0:
        raise WanAttnError(call, status)


def _stream_ptr(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_bshd(name, t, shape=None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
    if t.dim() != 4 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous [B, S, H, D] tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def fwd(q, k, v, o=None, lse=None, stream=None):
    """O, LSE = attention(q, k, v) through ``wan_attn_fwd``; outputs allocated if not given."""
    import torch
    _check_bshd("q", q)
    B, S, H, D = q.shape
    _check_bshd("k", k, q.shape)
    _check_bshd("v", v, q.shape)
    if o is None:
        o = torch.empty_like(q)
    _check_bshd("o", o, q.shape)
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, S) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 [B, H, S] tensor")
    _check("wan_attn_fwd", lib().wan_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                              lse.data_ptr(), B, S, H, D, _stream_ptr(stream)))
    return o, lse


def bwd_workspace_size(B, S, H, D=128) -> int:
    return lib().wan_attn_bwd_workspace_size(B, S, H, D)


def bwd(q, k, v, o, do, lse, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """dQ, dK, dV of sum(O * dO) through ``wan_attn_bwd``; outputs/workspace allocated if not given."""
    import torch
    _check_bshd("q", q)
    B, S, H, D = q.shape
    for name, t in (("k", k), ("v", v), ("o", o), ("do", do)):
        _check_bshd(name, t, q.shape)
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, S) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 [B, H, S] tensor")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _check_bshd(name, t, q.shape)
    need = bwd_workspace_size(B, S, H, D)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check("wan_attn_bwd", lib().wan_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                              do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                              dv.data_ptr(), B, S, H, D, workspace.data_ptr(),
                                              workspace.numel() * workspace.element_size(), _stream_ptr(stream)))
    return dq, dk, dv


def _check_kv(q, k, v):
    """K and V of a cross-attention call: [B, Skv, H, D] with q's B, H, D."""
    _check_bshd("k", k)
    B, _, H, D = q.shape
    Skv = k.shape[1]
    if (k.shape[0], k.shape[2], k.shape[3]) != (B, H, D):
        raise ValueError(f"k has shape {tuple(k.shape)}, expected [B={B}, Skv, H={H}, D={D}]")
    _check_bshd("v", v, k.shape)
    return Skv


def cross_fwd(q, k, v, o=None, lse=None, stream=None):
    """O, LSE of q [B, Sq, H, D] attending to k, v [B, Skv, H, D] through ``wan_attn_cross_fwd``."""
    import torch
    _check_bshd("q", q)
    B, Sq, H, D = q.shape
    Skv = _check_kv(q, k, v)
    o = torch.empty_like(q) if o is None else o
    _check_bshd("o", o, q.shape)
    if lse is None:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, Sq) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 [B, H, Sq] tensor")
    _check("wan_attn_cross_fwd", lib().wan_attn_cross_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                                          lse.data_ptr(), B, Sq, Skv, H, D, _stream_ptr(stream)))
    return o, lse


def block_sparse_workspace_size(B, Sq, Skv, H, D=128) -> int:
    return lib().wan_attn_fwd_block_sparse_workspace_size(B, Sq, Skv, H, D)


def fwd_block_sparse(q, k, v, block_mask, o=None, lse=None, workspace=None, stream=None):
    """O, LSE of q attending, per 64-token query block, only the 64-token key blocks that
    block_mask (uint8 [B, H, ceil(Sq/64), ceil(Skv/64)]) allows (``wan_attn_fwd_block_sparse``)."""
    import torch
    _check_bshd("q", q)
    B, Sq, H, D = q.shape
    Skv = _check_kv(q, k, v)
    nqb, nkb = (Sq + 63) // 64, (Skv + 63) // 64
    _check_plain("block_mask", block_mask, torch.uint8, B * H * nqb * nkb)
    o = torch.empty_like(q) if o is None else o
    _check_bshd("o", o, q.shape)
    if lse is None:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, Sq) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 [B, H, Sq] tensor")
    if workspace is None:
        workspace = torch.empty(block_sparse_workspace_size(B, Sq, Skv, H, D), dtype=torch.uint8, device=q.device)
    _check("wan_attn_fwd_block_sparse",
           lib().wan_attn_fwd_block_sparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                           block_mask.data_ptr(), B, Sq, Skv, H, D, workspace.data_ptr(),
                                           workspace.numel() * workspace.element_size(), _stream_ptr(stream)))
    return o, lse


def cross_bwd_workspace_size(B, Sq, Skv, H, D=128) -> int:
    return lib().wan_attn_cross_bwd_workspace_size(B, Sq, Skv, H, D)


def cross_bwd(q, k, v, o, do, lse, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """dQ, dK, dV of sum(O * dO) for the cross-attention through ``wan_attn_cross_bwd``."""
    import torch
    _check_bshd("q", q)
    B, Sq, H, D = q.shape
    Skv = _check_kv(q, k, v)
    for name, t in (("o", o), ("do", do)):
        _check_bshd(name, t, q.shape)
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, Sq) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 [B, H, Sq] tensor")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_bshd("dq", dq, q.shape)
    _check_bshd("dk", dk, k.shape)
    _check_bshd("dv", dv, k.shape)
    if workspace is None:
        workspace = torch.empty(cross_bwd_workspace_size(B, Sq, Skv, H, D), dtype=torch.uint8, device=q.device)
    _check("wan_attn_cross_bwd",
           lib().wan_attn_cross_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                                    lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Sq, Skv, H, D,
                                    workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                    _stream_ptr(stream)))
    return dq, dk, dv


CP_SEQ_TO_SEND, CP_RECV_TO_HEADS, CP_HEADS_TO_SEND, CP_RECV_TO_SEQ = 0, 1, 2, 3


def _check_plain(name, t, dtype, numel=None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous CUDA {dtype} tensor")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} has {t.numel()} elements, expected {numel}")


def cp_merge(o_acc, lse_acc, o_part, lse_part, first, o_out=None, stream=None):
    """Fold a partial (o_part bf16 [B, S, H, D], lse_part fp32 [B, H, S]) into the fp32 running
    (o_acc, lse_acc) through ``wan_attn_cp_merge``; o_out (bf16) receives the result if given."""
    import torch
    _check_bshd("o_part", o_part)
    B, S, H, D = o_part.shape
    _check_plain("o_acc", o_acc, torch.float32, o_part.numel())
    _check_plain("lse_acc", lse_acc, torch.float32, B * H * S)
    _check_plain("lse_part", lse_part, torch.float32, B * H * S)
    if o_out is not None:
        _check_bshd("o_out", o_out, o_part.shape)
    _check("wan_attn_cp_merge", lib().wan_attn_cp_merge(o_acc.data_ptr(), lse_acc.data_ptr(), o_part.data_ptr(),
                                                        lse_part.data_ptr(), o_out.data_ptr() if o_out is not None
                                                        else None, B, S, H, D, 1 if first else 0,
                                                        _stream_ptr(stream)))


def cp_accumulate(acc, part, first, out=None, stream=None):
    """acc (fp32) = (0 if first else acc) + part (bf16); out = bf16(acc) if given."""
    import torch
    _check_plain("part", part, torch.bfloat16)
    _check_plain("acc", acc, torch.float32, part.numel())
    if out is not None:
        _check_plain("out", out, torch.bfloat16, part.numel())
    _check("wan_attn_cp_accumulate", lib().wan_attn_cp_accumulate(acc.data_ptr(), part.data_ptr(),
                                                                  out.data_ptr() if out is not None else None,
                                                                  part.numel(), 1 if first else 0,
                                                                  _stream_ptr(stream)))


def cp_layout(dst, src, B, S_loc, G, Hg, which, D=128, stream=None):
    """Permute [Hg x D] blocks between the Ulysses orders (CP_* constants) through ``wan_attn_cp_layout``."""
    import torch
    n = B * S_loc * G * Hg * D
    _check_plain("src", src, torch.bfloat16, n)
    _check_plain("dst", dst, torch.bfloat16, n)
    _check("wan_attn_cp_layout", lib().wan_attn_cp_layout(dst.data_ptr(), src.data_ptr(), B, S_loc, G, Hg, D, which,
                                                          _stream_ptr(stream)))


def fp8_quantize_rows(x, codes=None, scales=None, stream=None):
    """Per-token e4m3 codes (uint8 [M, K]) and fp32 scales [M] of bf16 x [M, K] (``wan_fp8_quantize_rows``)."""
    import torch
    _check_plain("x", x, torch.bfloat16)
    if x.dim() != 2:
        raise ValueError("x must be [M, K]")
    M, K = x.shape
    codes = torch.empty((M, K), dtype=torch.uint8, device=x.device) if codes is None else codes
    scales = torch.empty(M, dtype=torch.float32, device=x.device) if scales is None else scales
    _check_plain("codes", codes, torch.uint8, M * K)
    _check_plain("scales", scales, torch.float32, M)
    _check("wan_fp8_quantize_rows", lib().wan_fp8_quantize_rows(x.data_ptr(), codes.data_ptr(), scales.data_ptr(),
                                                                M, K, _stream_ptr(stream)))
    return codes, scales


def fp8_quantize_tensor(w, codes=None, scale2=None, stream=None):
    """Per-tensor e4m3 codes (uint8 [N, K]) of bf16 w [N, K]; scale2 fp32 [2] = (sw, absmax)."""
    import torch
    _check_plain("w", w, torch.bfloat16)
    if w.dim() != 2:
        raise ValueError("w must be [N, K]")
    N, K = w.shape
    codes = torch.empty((N, K), dtype=torch.uint8, device=w.device) if codes is None else codes
    scale2 = torch.empty(2, dtype=torch.float32, device=w.device) if scale2 is None else scale2
    _check_plain("codes", codes, torch.uint8, N * K)
    _check_plain("scale2", scale2, torch.float32, 2)
    _check("wan_fp8_quantize_tensor", lib().wan_fp8_quantize_tensor(w.data_ptr(), codes.data_ptr(),
                                                                    scale2.data_ptr(), N, K, _stream_ptr(stream)))
    return codes, scale2


def fp8_gemm(a_codes, a_scales, b_codes, b_scale, y=None, stream=None):
    """bf16 Y [M, N] = diag(a_scales) (a_codes b_codes^T) b_scale[0] through ``wan_fp8_gemm``."""
    import torch
    _check_plain("a_codes", a_codes, torch.uint8)
    _check_plain("b_codes", b_codes, torch.uint8)
    if a_codes.dim() != 2 or b_codes.dim() != 2 or a_codes.shape[1] != b_codes.shape[1]:
        raise ValueError("a_codes [M, K] and b_codes [N, K] must share K")
    M, K = a_codes.shape
    N = b_codes.shape[0]
    _check_plain("a_scales", a_scales, torch.float32, M)
    _check_plain("b_scale", b_scale, torch.float32)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=a_codes.device) if y is None else y
    _check_plain("y", y, torch.bfloat16, M * N)
    _check("wan_fp8_gemm", lib().wan_fp8_gemm(a_codes.data_ptr(), a_scales.data_ptr(), b_codes.data_ptr(),
                                              b_scale.data_ptr(), y.data_ptr(), M, N, K, _stream_ptr(stream)))
    return y


def fp8_linear(x, w_codes, w_scale, stream=None):
    """Y = the FP8 linear layer of bf16 activations x [M, K] with a weight already quantised
    by fp8_quantize_tensor: the per-token quantiser, then the GEMM."""
    codes, scales = fp8_quantize_rows(x, stream=stream)
    return fp8_gemm(codes, scales, w_codes, w_scale, stream=stream)


def fwd_q8_workspace_size(B, S, H, D=128) -> int:
    return lib().wan_attn_fwd_q8_workspace_size(B, S, H, D)


def fwd_q8(q, k, v, o=None, lse=None, workspace=None, stream=None):
    """O, LSE of the 8-bit forward through ``wan_attn_fwd_q8``; returns (o, lse, workspace)."""
    import torch
    _check_bshd("q", q)
    B, S, H, D = q.shape
    _check_bshd("k", k, q.shape)
    _check_bshd("v", v, q.shape)
    o = torch.empty_like(q) if o is None else o
    _check_bshd("o", o, q.shape)
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, S) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 [B, H, S] tensor")
    if workspace is None:
        workspace = torch.empty(fwd_q8_workspace_size(B, S, H, D), dtype=torch.uint8, device=q.device)
    _check("wan_attn_fwd_q8", lib().wan_attn_fwd_q8(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                                    lse.data_ptr(), B, S, H, D, workspace.data_ptr(),
                                                    workspace.numel() * workspace.element_size(),
                                                    _stream_ptr(stream)))
    return o, lse, workspace


def q8_workspace_views(workspace, B, S, H, D=128):
    """Views of a wan_attn_fwd_q8 workspace: (q8, k8, v8 as uint8 [B, H, S, D], sq, sk, sv fp32 [B, H, nblk])."""
    import torch
    n = B * S * H * D
    nblk = (S + 63) // 64
    a = lambda x: (x + 255) // 256 * 256
    cb, sb = a(n), a(B * H * nblk * 4)
    codes = [workspace[i * cb:i * cb + n].view(B, H, S, D) for i in range(3)]
    scales = [workspace[3 * cb + i * sb:3 * cb + i * sb + B * H * nblk * 4].view(torch.float32).view(B, H, nblk)
              for i in range(3)]
    return (*codes, *scales)


def sync_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return lib().wan_attn_sync_status(_stream_ptr(stream))


def check_status(stream=None):
    _check("wan_attn_sync_status", sync_status(stream))


def set_wait_budget_ns(ns: int) -> int:
    return lib().wan_attn_set_wait_budget_ns(ns)


def selftest_wait_timeout(budget_ns: int, stream=None):
    _check("wan_attn_selftest_wait_timeout", lib().wan_attn_selftest_wait_timeout(budget_ns, _stream_ptr(stream)))
