"""Helpers for the GPU parity tests: move the seeded host inputs to the device
and measure errors against the oracle."""
import os

import numpy as np

import synth


def to_device(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_to_f64(t):
    """bf16 CUDA tensor -> fp64 numpy (exact)."""
    import torch
    return t.float().cpu().numpy().astype(np.float64)


def errors(got, want):
    """(max-abs error, relative Frobenius error)."""
    d = got - want
    return float(np.abs(d).max()), float(np.linalg.norm(d) / np.linalg.norm(want))


def inputs_for(B, S, H, D=128, seed=0, with_do=False, q_mul=1.0):
    shape = (B, S, H, D)
    x = {"q": synth.make_tensor(shape, seed, synth.STREAM_Q),
         "k": synth.make_tensor(shape, seed, synth.STREAM_K),
         "v": synth.make_tensor(shape, seed, synth.STREAM_V)}
    if q_mul != 1.0:
        f = synth.bf16_bits_to_f32(x["q"]) * np.float32(q_mul)
        x["q"] = synth.f64_to_bf16_bits(f.astype(np.float64))
    if with_do:
        x["do"] = synth.make_tensor(shape, seed, synth.STREAM_DO)
    return x


def inputs_for_cross(B, Sq, Skv, H, D=128, seed=0, with_do=False):
    """Q (and dO) [B, Sq, H, D], K and V [B, Skv, H, D] from the seeded generator."""
    x = {"q": synth.make_tensor((B, Sq, H, D), seed, synth.STREAM_Q),
         "k": synth.make_tensor((B, Skv, H, D), seed, synth.STREAM_K),
         "v": synth.make_tensor((B, Skv, H, D), seed, synth.STREAM_V)}
    if with_do:
        x["do"] = synth.make_tensor((B, Sq, H, D), seed, synth.STREAM_DO)
    return x


def oracle_bwd_by_head(x, q_rows, k_rows, heads, workers=None):
    """``oracle.attn_bwd`` evaluated one head per thread and stacked along the head axis.

    Heads are independent in the definition, and numpy's BLAS and ufuncs release the
    GIL, so threads scale; each thread's BLAS is held to one core.  Key rows need the
    LSE and D_i of every query row of their head (a full fp64 forward per head), which
    is what makes the large backward checks expensive."""
    from concurrent.futures import ThreadPoolExecutor

    from threadpoolctl import threadpool_limits

    import oracle
    heads = list(heads)
    workers = min(len(heads), workers or os.cpu_count() or 1)

    def one(h):
        return oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], q_rows=q_rows, k_rows=k_rows, heads=[h])

    with threadpool_limits(1), ThreadPoolExecutor(workers) as ex:
        parts = list(ex.map(one, heads))
    return {n: np.concatenate([p[n] for p in parts], axis=2 if n in ("dq", "dk", "dv") else 1)
            for n in parts[0]}
