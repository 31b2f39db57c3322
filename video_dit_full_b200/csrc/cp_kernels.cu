// Kernels of the context-parallel attention schemes the pages name for long sequences:
// kwkr.cn Wan explainer, section 3.2 (the token sequence is split over GPUs and the
// attention results are combined with Ulysses and Ring Attention), and "Wan: Open and
// Advanced Large-Scale Video Generative Models", section 5 (systems table: the DiT uses
// FSDP + 2-D context parallel, with layouts converted at module boundaries).  All three
// are HBM-bound elementwise / permutation kernels (grid-stride, 16-byte vector accesses,
// grids of 8 blocks per SM):
//
//   cp_merge      Ring Attention: fold one partial result (O_t, lse_t) of the queries
//                 against one key block into an fp32 running (O, lse):
//                     lse' = logaddexp(lse, lse_t)
//                     O'   = exp(lse - lse') O + exp(lse_t - lse') O_t
//                 which is exact: softmax over the union of key blocks.
//   cp_accumulate acc (+)= part (bf16 -> fp32), optionally writing bf16(acc): the ring
//                 backward's dQ and travelling dK, dV sums.
//   cp_layout     Ulysses: the permutations of [tokens x head groups] blocks around the
//                 all-to-alls that turn a sequence shard into a head shard and back.
#include "sm100_ptx.cuh"
#include "wan_attn_internal.h"

namespace wan {
namespace cp {

constexpr int HD = 128;

__device__ __forceinline__ float logaddexp(float a, float b) {
    const float m = fmaxf(a, b);
    return m + log1pf(__expf(-fabsf(a - b)));
}

// One half-warp (16 threads x 8 elements) per (b, s, h) row of 128.
__global__ void __launch_bounds__(256) cp_merge_kernel(float* __restrict__ o_acc, float* __restrict__ lse_acc,
                                                       const __nv_bfloat16* __restrict__ o_part,
                                                       const float* __restrict__ lse_part,
                                                       __nv_bfloat16* __restrict__ o_out, long long rows, int S,
                                                       int H, int first) {
    const long long total = rows * 16;
    const int lane = threadIdx.x & 31;
    const long long warp0 = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x - lane;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long t0 = warp0; t0 < total; t0 += stride) {          // warp-uniform trip count
        const long long t = t0 + lane;
        const bool valid = t < total;
        const long long r = valid ? (t >> 4) : 0;                    // row over [B, S, H]
        const int part = static_cast<int>(t & 15);
        // the row's first lane reads and updates the lse pair (the only lane that needs the
        // [B, H, S] index); its half-warp gets the weights
        float w_acc = 0.f, w_part = 1.f;
        if (valid && part == 0) {
            const long long h = r % H, bs = r / H, s = bs % S, b = bs / S;
            const long long li = (b * H + h) * S + s;
            const float lp = lse_part[li];
            if (first) {
                lse_acc[li] = lp;
            } else {
                const float la = lse_acc[li];
                const float ln = logaddexp(la, lp);
                w_acc = __expf(la - ln);
                w_part = __expf(lp - ln);
                lse_acc[li] = ln;
            }
        }
        w_acc = __shfl_sync(0xffffffffu, w_acc, lane & 16);
        w_part = __shfl_sync(0xffffffffu, w_part, lane & 16);
        if (valid) {
            const uint4 pv = *reinterpret_cast<const uint4*>(o_part + r * HD + part * 8);
            const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&pv);
            float4* acc4 = reinterpret_cast<float4*>(o_acc + r * HD + part * 8);
            float v[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(p2[e]);
                v[2 * e] = f.x * w_part;
                v[2 * e + 1] = f.y * w_part;
            }
            if (!first) {
                const float4 a0 = acc4[0], a1 = acc4[1];
                v[0] = fmaf(a0.x, w_acc, v[0]); v[1] = fmaf(a0.y, w_acc, v[1]);
                v[2] = fmaf(a0.z, w_acc, v[2]); v[3] = fmaf(a0.w, w_acc, v[3]);
                v[4] = fmaf(a1.x, w_acc, v[4]); v[5] = fmaf(a1.y, w_acc, v[5]);
                v[6] = fmaf(a1.z, w_acc, v[6]); v[7] = fmaf(a1.w, w_acc, v[7]);
            }
            acc4[0] = make_float4(v[0], v[1], v[2], v[3]);
            acc4[1] = make_float4(v[4], v[5], v[6], v[7]);
            if (o_out) {
                uint4 ov;
                ov.x = pack_bf16x2(v[0], v[1]);
                ov.y = pack_bf16x2(v[2], v[3]);
                ov.z = pack_bf16x2(v[4], v[5]);
                ov.w = pack_bf16x2(v[6], v[7]);
                *reinterpret_cast<uint4*>(o_out + r * HD + part * 8) = ov;
            }
        }
    }
}

// acc (+)= part for n8 groups of 8 elements; out = bf16(acc) when given.
__global__ void __launch_bounds__(256) cp_accumulate_kernel(float* __restrict__ acc,
                                                            const __nv_bfloat16* __restrict__ part,
                                                            __nv_bfloat16* __restrict__ out, long long n8,
                                                            int first) {
    const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long t = tid; t < n8; t += stride) {
        const uint4 pv = reinterpret_cast<const uint4*>(part)[t];
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&pv);
        float v[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(p2[e]);
            v[2 * e] = f.x;
            v[2 * e + 1] = f.y;
        }
        float4* a4 = reinterpret_cast<float4*>(acc) + 2 * t;
        if (!first) {
            const float4 a0 = a4[0], a1 = a4[1];
            v[0] += a0.x; v[1] += a0.y; v[2] += a0.z; v[3] += a0.w;
            v[4] += a1.x; v[5] += a1.y; v[6] += a1.z; v[7] += a1.w;
        }
        a4[0] = make_float4(v[0], v[1], v[2], v[3]);
        a4[1] = make_float4(v[4], v[5], v[6], v[7]);
        if (out) {
            uint4 ov;
            ov.x = pack_bf16x2(v[0], v[1]);
            ov.y = pack_bf16x2(v[2], v[3]);
            ov.z = pack_bf16x2(v[4], v[5]);
            ov.w = pack_bf16x2(v[6], v[7]);
            reinterpret_cast<uint4*>(out)[t] = ov;
        }
    }
}

// Blocks of `blk16` 16-byte words (Hg * D bf16) indexed by (g, b, s) move between the four
// orders of the Ulysses exchange (see wan_attn.h: WAN_ATTN_CP_*).
__device__ __forceinline__ long long layout_src_block(int which, long long g, long long b, long long s, int G,
                                                      int B, int S) {
    switch (which) {
        case 0: return (b * S + s) * G + g;      // [B, S, G]
        case 1: return (g * B + b) * S + s;      // [G, B, S]
        case 2: return (b * G + g) * S + s;      // [B, G, S]
        default: return (g * B + b) * S + s;     // [G, B, S]
    }
}
__device__ __forceinline__ long long layout_dst_block(int which, long long g, long long b, long long s, int G,
                                                      int B, int S) {
    switch (which) {
        case 0: return (g * B + b) * S + s;      // [G, B, S]
        case 1: return (b * G + g) * S + s;      // [B, G, S]
        case 2: return (g * B + b) * S + s;      // [G, B, S]
        default: return (b * S + s) * G + g;     // [B, S, G]
    }
}

// One warp per block (grid-stride over blocks): the index arithmetic once per block, then
// the block's 16-byte words by the 32 lanes.
__global__ void __launch_bounds__(256) cp_layout_kernel(uint4* __restrict__ dst, const uint4* __restrict__ src,
                                                        int B, int S, int G, int blk16, int which) {
    const long long nblk = static_cast<long long>(G) * B * S;
    const int lane = threadIdx.x & 31;
    const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    for (long long k = warp; k < nblk; k += nwarps) {          // block index in (g, b, s) order
        const long long s = k % S, gb = k / S, b = gb % B, g = gb / B;
        uint4* d = dst + layout_dst_block(which, g, b, s, G, B, S) * blk16;
        const uint4* sp = src + layout_src_block(which, g, b, s, G, B, S) * blk16;
        for (int w = lane; w < blk16; w += 32) d[w] = sp[w];
    }
}

int ew_grid() {
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms * 8;
}

}  // namespace cp

int launch_cp_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, void* o_out, int B,
                    int S, int H, int first, cudaStream_t stream) {
    const long long rows = static_cast<long long>(B) * S * H;
    cp::cp_merge_kernel<<<cp::ew_grid(), 256, 0, stream>>>(o_acc, lse_acc,
                                                          static_cast<const __nv_bfloat16*>(o_part), lse_part,
                                                          static_cast<__nv_bfloat16*>(o_out), rows, S, H, first);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_cp_accumulate(float* acc, const void* part, void* out, long long n8, int first, cudaStream_t stream) {
    cp::cp_accumulate_kernel<<<cp::ew_grid(), 256, 0, stream>>>(acc, static_cast<const __nv_bfloat16*>(part),
                                                               static_cast<__nv_bfloat16*>(out), n8, first);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_cp_layout(void* dst, const void* src, int B, int S, int G, int blk16, int which, cudaStream_t stream) {
    cp::cp_layout_kernel<<<cp::ew_grid(), 256, 0, stream>>>(static_cast<uint4*>(dst), static_cast<const uint4*>(src),
                                                           B, S, G, blk16, which);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace wan
