"""Parity of the FP8 GEMM calls (wan_fp8_quantize_rows / _tensor, wan_fp8_gemm, through the C ABI)
with the oracle (oracle/fp8_gemm.py).

* Codes and scales are decided in fp32 on both sides: bit-exact.
* The GEMM against the oracle's fp64 product of its own code values: the only differences
  are the fp32 accumulation order and the bf16 rounding of Y (2^-9 relative), so the bar is
  relative Frobenius <= 5e-3 and max-abs <= 1e-2 of max |Y|.
* Shapes cover ragged M, N and K (zero-filled tiles), one row, and the 720p fused QKV
  projection (hidden 40 x 128 = 5120; N = 3 x 5120) on 256 sampled rows.
"""
import numpy as np
import pytest

import synth
from gpu_util import to_device
from oracle import fp8_gemm as fg

pytestmark = pytest.mark.gpu

REL_FROB, MAX_ABS_FRAC = 5e-3, 1e-2


def bits_of(t):
    return t.cpu().numpy()


def make(M, N, K, seed):
    x = synth.make_tensor((M, K), seed, synth.STREAM_Q)
    w = synth.make_tensor((N, K), seed, synth.STREAM_K)
    return x, w


@pytest.mark.parametrize("M,K", [(1, 16), (3, 48), (130, 144), (513, 5120)])
def test_row_quantiser_bit_exact(M, K):
    import video_dit_full_b200 as wa
    x = synth.make_tensor((M, K), M + K, synth.STREAM_Q)
    if M > 2:
        x[1] = 0                                   # an all-zero row: codes 0, scale 1
    codes, scales = wa.fp8_quantize_rows(to_device(x))
    wa.check_status()
    want_bits, _, want_s = fg.quant_rows(x)
    np.testing.assert_array_equal(bits_of(codes), want_bits)
    np.testing.assert_array_equal(scales.cpu().numpy(), want_s)


@pytest.mark.parametrize("N,K", [(8, 16), (264, 144), (5120, 5120)])
def test_tensor_quantiser_bit_exact(N, K):
    import video_dit_full_b200 as wa
    w = synth.make_tensor((N, K), N, synth.STREAM_K)
    codes, scale2 = wa.fp8_quantize_tensor(to_device(w))
    wa.check_status()
    want_bits, _, want_s = fg.quant_tensor(w)
    np.testing.assert_array_equal(bits_of(codes), want_bits)
    s = scale2.cpu().numpy()
    assert s[0] == want_s
    assert s[1] == np.abs(synth.bf16_bits_to_f32(w)).max()


def check_gemm(x, w, rows=None):
    import video_dit_full_b200 as wa
    wc, ws = wa.fp8_quantize_tensor(to_device(w))
    y = wa.fp8_linear(to_device(x), wc, ws[:1])
    wa.check_status()
    want = fg.fp8_linear(x, w, rows=rows)
    got = y.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        got = got[rows]
    d = got - want
    rel = np.linalg.norm(d) / np.linalg.norm(want)
    max_frac = np.abs(d).max() / np.abs(want).max()
    print(f"Y rel-frob {rel:.3e}  max-abs / max|Y| {max_frac:.3e}")
    assert np.all(np.isfinite(got))
    assert rel <= REL_FROB and max_frac <= MAX_ABS_FRAC, (rel, max_frac)


@pytest.mark.parametrize("M,N,K", [(1, 8, 16), (130, 264, 144), (300, 256, 256), (1000, 520, 1040),
                                   (128, 256, 5120), (257, 1032, 2064)])
def test_gemm_shapes_full(M, N, K):
    x, w = make(M, N, K, seed=M + N + K)
    check_gemm(x, w)


def test_gemm_720p_qkv_projection_sampled_rows():
    M, N, K = synth.tokens_for_video(81, 720, 1280), 3 * 40 * 128, 40 * 128
    x, w = make(M, N, K, seed=0)
    check_gemm(x, w, rows=synth.sample_rows(M, 256))
