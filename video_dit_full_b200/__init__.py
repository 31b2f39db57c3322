"""B200 (sm_100a) full spatio-temporal self-attention (and the text cross-attention) for Wan-style video DiTs.

The computation lives in ``libwan_attn.so`` (hand-written CUDA for sm_100a,
C ABI in ``include/wan_attn.h``); ``wan_attn`` is its ctypes binding.
"""
from .wan_attn import (CP_HEADS_TO_SEND, CP_RECV_TO_HEADS, CP_RECV_TO_SEQ, CP_SEQ_TO_SEND,  # noqa: F401
                       WanAttnError, bwd, bwd_workspace_size, check_status, cp_accumulate, cp_layout, cp_merge,
                       block_sparse_workspace_size, cross_bwd, cross_bwd_workspace_size, cross_fwd, fp8_gemm,
                       fp8_linear, fp8_quantize_rows, fwd_block_sparse,
                       fp8_quantize_tensor, fwd, fwd_q8, fwd_q8_workspace_size, lib,
                       q8_workspace_views, selftest_wait_timeout, set_wait_budget_ns, sync_status)
