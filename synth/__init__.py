"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This package holds no arithmetic of the attention method: it turns
(seed, stream, index) into numbers (``synth.c`` states the generator) and
describes the workloads' shapes.  Both the oracle and the GPU path read the
same host bytes that it writes.

Streams: 0 = Q, 1 = K, 2 = V, 3 = dO, 4 = peaky-head choice,
5 = sampled query rows, 6 = sampled key rows, 7 = block-sparse masks.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None

STREAM_Q, STREAM_K, STREAM_V, STREAM_DO = 0, 1, 2, 3
STREAM_PEAKY, STREAM_QROWS, STREAM_KROWS = 4, 5, 6
STREAM_MASK = 7


def build(force: bool = False) -> str:
    """Compile ``libsynth.so`` beside its source with gcc (a second or so)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-pthread", _SRC,
                               "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        u64 = ctypes.c_uint64
        lib.synth_key.restype = u64
        lib.synth_key.argtypes = [u64, u64]
        lib.synth_normal_bf16.restype = None
        lib.synth_normal_bf16.argtypes = [u64, u64, u64, u64, ctypes.c_void_p, ctypes.c_int]
        lib.synth_normal_f64.restype = None
        lib.synth_normal_f64.argtypes = [u64, u64, u64, u64, ctypes.c_void_p, ctypes.c_int]
        lib.synth_uniform_f64.restype = None
        lib.synth_uniform_f64.argtypes = [u64, u64, u64, u64, ctypes.c_void_p]
        _lib = lib
    return _lib


def _threads(nthreads):
    return int(nthreads or os.cpu_count() or 1)


def normal_bf16(seed: int, stream: int, n: int, first: int = 0, nthreads=None,
                out: np.ndarray | None = None) -> np.ndarray:
    """n standard normals of one stream (elements first..first+n-1) as bf16 bit patterns."""
    lib = _load()
    if out is None:
        out = np.empty(n, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous and out.size == n
    lib.synth_normal_bf16(seed, stream, first, n, out.ctypes.data, _threads(nthreads))
    return out


def normal_f64(seed: int, stream: int, n: int, first: int = 0, nthreads=None) -> np.ndarray:
    lib = _load()
    out = np.empty(n, dtype=np.float64)
    lib.synth_normal_f64(seed, stream, first, n, out.ctypes.data, _threads(nthreads))
    return out


def uniform(seed: int, stream: int, n: int, first: int = 0) -> np.ndarray:
    lib = _load()
    out = np.empty(n, dtype=np.float64)
    lib.synth_uniform_f64(seed, stream, first, n, out.ctypes.data)
    return out


# ---------------------------------------------------------------------------
# numpy twin of the generator (slow; used by the tests to check the C code)
# ---------------------------------------------------------------------------
_M64 = (1 << 64) - 1
_G = 0x9E3779B97F4A7C15


def _mix_int(z: int) -> int:
    z &= _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def key_py(seed: int, stream: int) -> int:
    return _mix_int(_mix_int(seed + _G) ^ ((stream * 0xD1B54A32D192ED03 + _G) & _M64))


def _mix_np(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def normal_f64_np(seed: int, stream: int, n: int, first: int = 0) -> np.ndarray:
    key = np.uint64(key_py(seed, stream))
    idx = np.arange(first, first + n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        x1 = _mix_np(key + (np.uint64(2) * idx + np.uint64(1)) * np.uint64(_G))
        x2 = _mix_np(key + (np.uint64(2) * idx + np.uint64(2)) * np.uint64(_G))
    u1 = 1.0 - (x1 >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    u2 = (x2 >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 (nearest even) -> bf16 (nearest even), as uint16 bit patterns."""
    u = np.asarray(x, dtype=np.float64).astype(np.float32).view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return u.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
def tokens_for_video(frames: int, height: int, width: int) -> int:
    """Token count of a (frames x height x width x 3) clip after the Wan-VAE
    (time /4 after the first frame, space /8, 16 channels) and the (1,2,2)
    patchify: (1 + (frames-1)/4) * (height/16) * (width/16).

    Wan 2.1 paper-podcast summary, section on attention cost ("先看现象");
    "Wan: Open and Advanced Large-Scale Video Generative Models", section 3
    (Wan-VAE compression formula).
    """
    if (frames - 1) % 4 or height % 16 or width % 16:
        raise ValueError("frames must be 1+4k and height/width multiples of 16")
    return (1 + (frames - 1) // 4) * (height // 16) * (width // 16)


TEXT_TOKENS = 512   # length of the umT5 text embedding the DiT cross-attends to


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    S: int
    H: int
    D: int
    video: tuple | None = None     # (frames, height, width) the token count comes from
    peaky_frac: float = 0.0        # fraction of heads whose Q is scaled x2
    backward: bool = False
    q8: bool = False
    Skv: int | None = None         # key/value tokens when they differ from S (cross-attention)
    cp: str | None = None          # "ring" / "ulysses": one rank's share of a G-way context split
    cp_ranks: int = 1
    gemm: tuple | None = None      # (M, N, K) of an FP8 linear layer instead of attention
    sparse_keep: float = 0.0       # block-sparse: fraction of 64-token key blocks each query block keeps

    @property
    def kv_len(self) -> int:
        return self.S if self.Skv is None else self.Skv

    @property
    def cross(self) -> bool:
        return self.Skv is not None

    @property
    def fwd_flop(self) -> float:
        """4*B*H*S*Skv*D: the forward's two S x Skv x D contractions (multiply-add = 2);
        for a context-parallel workload, one rank's 1/G share of it."""
        if self.gemm:
            M, N, K = self.gemm
            return 2.0 * M * N * K
        return 4.0 * self.B * self.H * self.S * self.kv_len * self.D / self.cp_ranks


WORKLOADS = {
    "oracle_1280": Workload("oracle_1280", 1, tokens_for_video(17, 256, 256), 12, 128,
                            video=(17, 256, 256)),
    "wan1.3b_480p_cfg": Workload("wan1.3b_480p_cfg", 2, tokens_for_video(81, 480, 832), 12, 128,
                                 video=(81, 480, 832), peaky_frac=0.1),
    "wan14b_720p": Workload("wan14b_720p", 1, tokens_for_video(81, 720, 1280), 40, 128,
                            video=(81, 720, 1280)),
    "train_480p_fwd_bwd": Workload("train_480p_fwd_bwd", 1, tokens_for_video(81, 480, 832), 40, 128,
                                   video=(81, 480, 832), backward=True),
    "q8_720p": Workload("q8_720p", 1, tokens_for_video(81, 720, 1280), 40, 128,
                        video=(81, 720, 1280), q8=True),
    # the DiT block's cross-attention: video-token queries against the 512-token umT5 text
    # embedding (Wan 2.1 paper-podcast summary, section "干预与形式化")
    "cross_720p": Workload("cross_720p", 1, tokens_for_video(81, 720, 1280), 40, 128,
                           video=(81, 720, 1280), Skv=TEXT_TOKENS),
    "cross_train_480p": Workload("cross_train_480p", 1, tokens_for_video(81, 480, 832), 40, 128,
                                 video=(81, 480, 832), backward=True, Skv=TEXT_TOKENS),
    # one rank's compute of the 720p attention split 8 ways (kwkr.cn Wan explainer, section 3.2)
    "ring8_720p_rank": Workload("ring8_720p_rank", 1, tokens_for_video(81, 720, 1280), 40, 128,
                                video=(81, 720, 1280), cp="ring", cp_ranks=8),
    "ulysses8_720p_rank": Workload("ulysses8_720p_rank", 1, tokens_for_video(81, 720, 1280), 40, 128,
                                   video=(81, 720, 1280), cp="ulysses", cp_ranks=8),
    # block-sparse attention keeping 1/8 of the 64 x 64 blocks (87.5 % sparsity, the FastWan /
    # VSA article on the first page), random seeded mask
    "sparse8_720p": Workload("sparse8_720p", 1, tokens_for_video(81, 720, 1280), 40, 128,
                             video=(81, 720, 1280), sparse_keep=0.125),
    # the DiT block's fused Q/K/V projection at 720p in FP8 (kwkr.cn Wan explainer, section 4.2):
    # tokens x hidden (40 x 128) -> 3 x hidden
    "fp8_qkv_720p": Workload("fp8_qkv_720p", 1, tokens_for_video(81, 720, 1280), 40, 128,
                             video=(81, 720, 1280),
                             gemm=(tokens_for_video(81, 720, 1280), 3 * 40 * 128, 40 * 128)),
}


def peaky_heads(H: int, frac: float, seed: int = 0) -> list:
    """Seeded choice of max(1, round(frac*H)) heads (stream 4): the heads with
    the smallest uniform draws, returned in ascending order."""
    if frac <= 0:
        return []
    k = max(1, int(round(frac * H)))
    u = uniform(seed, STREAM_PEAKY, H)
    return sorted(int(h) for h in np.argsort(u, kind="stable")[:k])


def sample_rows(S: int, n: int = 256, seed: int = 0, stream: int = STREAM_QROWS) -> np.ndarray:
    """n distinct token indices in [0, S): 0 and S-1 always, the rest the
    indices 1..S-2 with the smallest uniform draws of the stream.  All rows if S <= n."""
    if S <= n:
        return np.arange(S, dtype=np.int64)
    u = uniform(seed, stream, S)[1:S - 1]
    pick = np.argsort(u, kind="stable")[: n - 2] + 1
    return np.sort(np.concatenate([[0, S - 1], pick]).astype(np.int64))


def block_mask(B: int, H: int, nqb: int, nkb: int, keep: float, seed: int = 0) -> np.ndarray:
    """A 64 x 64 block mask uint8 [B, H, nqb, nkb] keeping max(1, round(keep * nkb)) key blocks
    per query block: those with the smallest uniform draws of stream 7 (row-major order)."""
    u = uniform(seed, STREAM_MASK, B * H * nqb * nkb).reshape(B, H, nqb, nkb)
    n = max(1, int(round(keep * nkb)))
    pick = np.argsort(u, axis=3, kind="stable")[..., :n]
    mask = np.zeros((B, H, nqb, nkb), dtype=np.uint8)
    np.put_along_axis(mask, pick, 1, axis=3)
    return mask


def make_tensor(shape, seed: int, stream: int, nthreads=None) -> np.ndarray:
    n = int(np.prod(shape))
    return normal_bf16(seed, stream, n, nthreads=nthreads).reshape(shape)


def make_inputs(w: Workload, seed: int = 0, with_do: bool | None = None, nthreads=None,
                S: int | None = None, Skv: int | None = None) -> dict:
    """Q, K, V (and dO) for a workload as bf16 bit patterns: Q (and dO) [B, S, H, D],
    K and V [B, Skv, H, D] (Skv = S for self-attention), row-major.

    ``S`` / ``Skv`` override the workload's query / key token counts (small parity cases)."""
    S = w.S if S is None else S
    if Skv is None:
        Skv = w.kv_len if w.cross else S
    shape = (w.B, S, w.H, w.D)
    kv_shape = (w.B, Skv, w.H, w.D)
    out = {"q": make_tensor(shape, seed, STREAM_Q, nthreads),
           "k": make_tensor(kv_shape, seed, STREAM_K, nthreads),
           "v": make_tensor(kv_shape, seed, STREAM_V, nthreads)}
    heads = peaky_heads(w.H, w.peaky_frac, seed)
    if heads:
        q = out["q"]
        for h in heads:   # x2 is exact in bf16 (exponent + 1) for these magnitudes
            f = bf16_bits_to_f32(q[:, :, h, :]) * np.float32(2.0)
            q[:, :, h, :] = (f.view(np.uint32) >> 16).astype(np.uint16)
    if with_do if with_do is not None else w.backward:
        out["do"] = make_tensor(shape, seed, STREAM_DO, nthreads)
    out["peaky_heads"] = heads
    return out
