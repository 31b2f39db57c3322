// FP8 GEMM of the DiT linear layers on sm_100a: Y = diag(sx) (Xq Wq^T) sw.
//
// The pages: kwkr.cn Wan explainer, section 4.2 (the most expensive matrix products
// run in FP8, weights quantised per tensor and activations per token), and the Wan
// 2.1 paper-podcast summary, section "干预与形式化" (FP8 GEMM, 1.13x).
//
// Three kernels:
//   fp8_quant_rows     X [M, K] bf16 -> e4m3 codes and one fp32 scale per row (token):
//                      sx = absmax / 448, codes = e4m3(fp32(x * fp32(448 / absmax))).
//   fp8_absmax /       W [N, K] bf16 -> its absmax (atomic max of the bit patterns of
//   fp8_quant_tensor   non-negative floats), then e4m3 codes with the one per-tensor scale.
//   fp8_gemm_kernel    persistent, one CTA per SM walking 128 x 256 output tiles (in groups of
//                      16 row blocks, the row block fastest, so the tiles in flight share
//                      a few row blocks of X and column blocks of W in L2):
//                        warp 0      TMA: [128 x 128 B] of X and [256 x 128 B] of W per stage,
//                                    4 stages, 128-byte swizzle, zero fill past the edges
//                        warp 1      tcgen05.mma kind::f8f6f4 (e4m3 x e4m3 -> fp32), M128 N256
//                                    K32, into one of two 256-column TMEM accumulators
//                        warps 2-5   epilogue: TMEM -> y = acc * sx[m] * sw -> bf16 -> global,
//                                    overlapping the next tile's main loop (TMEM ping-pong)
//   fp8_gemm_pair_kernel the same on 2-CTA clusters (tcgen05 cta_group::2, 256 x 256 tiles),
//                      used when M > 128: each CTA stages only half of W's tile rows.
#include <cuda.h>

#include "sm100_ptx.cuh"
#include "wan_attn_internal.h"

namespace wan {
namespace fp8 {

constexpr float E4M3_MAX = 448.f;

// One warp per row (grid-stride).  K % 16 == 0: 8 bf16 per lane per 16-byte load.
__global__ void __launch_bounds__(256) fp8_quant_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                             uint8_t* __restrict__ codes,
                                                             float* __restrict__ scales, int M, int K) {
    const int lane = threadIdx.x & 31;
    const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    const int k8 = K / 8;
    for (long long m = warp; m < M; m += nwarps) {
        const uint4* row = reinterpret_cast<const uint4*>(x + m * K);
        float amax = 0.f;
        for (int c = lane; c < k8; c += 32) {
            const uint4 u = row[c];
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h[e]);
                amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        float inv = 1.f, scale = 1.f;
        if (amax > 0.f) {
            inv = __fdiv_rn(E4M3_MAX, amax);
            scale = __fdiv_rn(amax, E4M3_MAX);
        }
        if (lane == 0) scales[m] = scale;
        uint2* out = reinterpret_cast<uint2*>(codes + m * K);
        for (int c = lane; c < k8; c += 32) {
            const uint4 u = row[c];
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
            uint32_t w[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float2 a = __bfloat1622float2(h[2 * e]);
                const float2 b = __bfloat1622float2(h[2 * e + 1]);
                w[e] = pack_e4m3x2(__fmul_rn(a.x, inv), __fmul_rn(a.y, inv)) |
                       (pack_e4m3x2(__fmul_rn(b.x, inv), __fmul_rn(b.y, inv)) << 16);
            }
            out[c] = make_uint2(w[0], w[1]);
        }
    }
}

// absmax of n8 groups of 8 bf16 into *amax_bits (a float's bits; zeroed by the caller).
__global__ void __launch_bounds__(256) fp8_absmax_kernel(const __nv_bfloat16* __restrict__ w, long long n8,
                                                         unsigned int* __restrict__ amax_bits) {
    const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    float amax = 0.f;
    for (long long t = tid; t < n8; t += stride) {
        const uint4 u = reinterpret_cast<const uint4*>(w)[t];
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h[e]);
            amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(amax));   // non-negative: bits order
}

// codes = e4m3(w * fp32(448 / absmax)); block 0 also writes the scale absmax / 448.
__global__ void __launch_bounds__(256) fp8_quant_tensor_kernel(const __nv_bfloat16* __restrict__ w,
                                                               uint8_t* __restrict__ codes, long long n8,
                                                               const unsigned int* __restrict__ amax_bits,
                                                               float* __restrict__ scale_out) {
    const float amax = __uint_as_float(*amax_bits);
    float inv = 1.f, scale = 1.f;
    if (amax > 0.f) {
        inv = __fdiv_rn(E4M3_MAX, amax);
        scale = __fdiv_rn(amax, E4M3_MAX);
    }
    const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (tid == 0) *scale_out = scale;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long t = tid; t < n8; t += stride) {
        const uint4 u = reinterpret_cast<const uint4*>(w)[t];
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
        uint32_t o[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float2 a = __bfloat1622float2(h[2 * e]);
            const float2 b = __bfloat1622float2(h[2 * e + 1]);
            o[e] = pack_e4m3x2(__fmul_rn(a.x, inv), __fmul_rn(a.y, inv)) |
                   (pack_e4m3x2(__fmul_rn(b.x, inv), __fmul_rn(b.y, inv)) << 16);
        }
        reinterpret_cast<uint2*>(codes)[t] = make_uint2(o[0], o[1]);
    }
}

// ------------------------------------------------------------------------------------
// GEMM
// ------------------------------------------------------------------------------------
constexpr int BM = 128, BN = 256, BK = 128;          // BK in bytes = e4m3 elements
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK, B_BYTES = BN * BK, STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int OFF_BAR = STAGES * STAGE_BYTES;
enum Bar { FULL = 0, EMPTY = STAGES, TFULL = 2 * STAGES, TEMPTY = 2 * STAGES + 2, DRAIN = 2 * STAGES + 4,
           NBARS = 2 * STAGES + 5 };
constexpr int OFF_TMEM_SLOT = OFF_BAR + NBARS * 8;
constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
constexpr int SMEM_BYTES = OFF_ABORT + 8 + 1024;
constexpr int NTHREADS = 192;                       // warp 0 TMA, 1 MMA, 2-5 epilogue
constexpr uint32_t TMEM_COLS = 512;                 // two 256-column fp32 accumulators
#ifndef FP8_GROUP_M
#define FP8_GROUP_M 16
#endif
constexpr int GROUP_M = FP8_GROUP_M;                // tile order: row blocks in groups of GROUP_M

// Tile t -> (row block, column block): the tiles are walked in groups of GROUP_M row blocks,
// the row block varying fastest inside a group.  The CTAs at work at any moment then share a
// few row blocks of X and a few column blocks of W, which stay in L2.
__device__ __forceinline__ void tile_of(long long t, int m_tiles, int n_tiles, int& mb, int& nb) {
    const long long per_group = static_cast<long long>(GROUP_M) * n_tiles;
    const int g = static_cast<int>(t / per_group);
    const int rows = min(GROUP_M, m_tiles - g * GROUP_M);
    const long long w = t - g * per_group;
    mb = g * GROUP_M + static_cast<int>(w % rows);
    nb = static_cast<int>(w / rows);
}

__global__ void __launch_bounds__(NTHREADS, 1)
fp8_gemm_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                const Fp8GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_addr);
    const int warp = warp_id(), lane = lane_id();
    const uint32_t bar0 = base + OFF_BAR;
    auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
    const WaitCtl wc{abort_flag, p.wait_budget_ns, p.status};

    const int m_tiles = (p.M + BM - 1) / BM, n_tiles = (p.N + BN - 1) / BN;
    const long long tiles = static_cast<long long>(m_tiles) * n_tiles;
    const int nk = (p.K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar(FULL + s), 1);
            mbar_init(bar(EMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(TFULL + b), 1);
            mbar_init(bar(TEMPTY + b), 128);
        }
        mbar_init(bar(DRAIN), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(base + OFF_TMEM_SLOT, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEM_SLOT);

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&tma_a);
            tma_prefetch_desc(&tma_b);
            int par[STAGES];
            for (int s = 0; s < STAGES; ++s) par[s] = -1;
            long long it = 0;
            bool ok = true;
            for (long long t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                int mb, nbk;
                tile_of(t, m_tiles, n_tiles, mb, nbk);
                const int m0 = mb * BM, n0 = nbk * BN;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = static_cast<int>(it % STAGES);
                    const int use = static_cast<int>((it / STAGES) & 1);
                    ok = wait_thread(bar(EMPTY + s), use ^ 1, wc);
                    if (!ok) break;
                    const uint32_t st = base + s * STAGE_BYTES;
                    mbar_arrive_expect_tx(bar(FULL + s), STAGE_BYTES);
                    tma_load_2d(st, &tma_a, bar(FULL + s), kb * BK, m0);
                    tma_load_2d(st + A_BYTES, &tma_b, bar(FULL + s), kb * BK, n0);
                    par[s] = use;
                }
            }
            if (!ok)
                for (int s = 0; s < STAGES; ++s)
                    if (par[s] >= 0) drain_wait(bar(FULL + s), par[s]);
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0) {
            const uint32_t idesc = make_idesc(1, 0, 0, 0, 0, BM, BN);   // f32 <- e4m3 x e4m3, K-major
            long long it = 0;
            int tc = 0;
            bool ok = true;
            for (long long t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++tc) {
                const int b = tc & 1;
                ok = wait_thread(bar(TEMPTY + b), ((tc >> 1) & 1) ^ 1, wc);
                if (!ok) break;
                tc_fence_after();
                const uint32_t acc = tmem + b * BN;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = static_cast<int>(it % STAGES);
                    ok = wait_thread(bar(FULL + s), static_cast<int>((it / STAGES) & 1), wc);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t sa = base + s * STAGE_BYTES, sb = sa + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk)        // K = 32 e4m3 = 32 bytes per MMA
                        mma_f8_ss(acc, sdesc_sw128(sa + kk * 32, 16, 1024), sdesc_sw128(sb + kk * 32, 16, 1024),
                                  idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(bar(EMPTY + s));                  // the stage is free once these finish
                }
                if (!ok) break;
                mma_commit(bar(TFULL + b));
            }
            mma_commit(bar(DRAIN));
            drain_wait(bar(DRAIN), 0);
        }
    } else {
        // ------------------------------ epilogue ----------------------------------
        const int r = (warp & 3) * 32 + lane;                  // TMEM lane = row of the tile
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const float sw = *p.b_scale;
        int tc = 0;
        bool ok = true;
        for (long long t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++tc) {
            int mb, nbk;
            tile_of(t, m_tiles, n_tiles, mb, nbk);
            const int m0 = mb * BM, n0 = nbk * BN;
            const int b = tc & 1;
            ok = wait_warp(bar(TFULL + b), (tc >> 1) & 1, wc);
            if (!ok) break;
            tc_fence_after();
            const int m = m0 + r;
            const bool row_ok = m < p.M;
            const float sc = row_ok ? p.a_scales[m] * sw : 0.f;
            __nv_bfloat16* yrow = reinterpret_cast<__nv_bfloat16*>(p.y) + static_cast<long long>(m) * p.N;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem + b * BN + lane_off + c * 32, v);
                tmem_wait_ld();
                const int n = n0 + c * 32;
                if (row_ok && n < p.N) {
                    uint4 pk[4];
                    uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pw[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * sc, __uint_as_float(v[2 * e + 1]) * sc);
                    uint4* dst = reinterpret_cast<uint4*>(yrow + n);
#pragma unroll
                    for (int q = 0; q < 4; ++q)                  // N % 8 == 0: whole 16-byte chunks
                        if (n + q * 8 < p.N) dst[q] = pk[q];
                }
            }
            tc_fence_before();
            mbar_arrive(bar(TEMPTY + b));                         // the accumulator may be reused
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

// ------------------------------------------------------------------------------------
// The same GEMM on CTA pairs (tcgen05 cta_group::2): a pair computes a 256 x 256 tile.  CTA r
// (its rank in the 2-CTA cluster) loads rows m0 + 128 r of X and rows n0 + 128 r of W (half of
// the tile's B) into its own shared memory; the leader (r = 0) issues M256 N256 K32 MMAs that
// read both CTAs' operands, each CTA's TMEM receiving its own 128 rows of the accumulator.  Per
// CTA that is half the B bytes of the 1-CTA kernel, loaded by TMA and read by the tensor core.
// Barriers: FULL (leader's, counting both CTAs' TMA bytes), EMPTY and TFULL (in each CTA,
// signalled by the leader's commits), TEMPTY (leader's, 128 arrivals from each CTA).
// ------------------------------------------------------------------------------------
#ifndef FP8_PAIR_STAGES
#define FP8_PAIR_STAGES 6
#endif
constexpr int STAGES2 = FP8_PAIR_STAGES;            // 32 KB each
constexpr int HALF_BYTES = 128 * BK, STAGE2_BYTES = 2 * HALF_BYTES;    // A rows | B half rows
constexpr int OFF_BAR2 = STAGES2 * STAGE2_BYTES;
enum Bar2 { F2 = 0, E2 = STAGES2, TF2 = 2 * STAGES2, TE2 = 2 * STAGES2 + 2, DR2 = 2 * STAGES2 + 4,
            NBARS2 = 2 * STAGES2 + 5 };
constexpr int OFF_TMEM_SLOT2 = OFF_BAR2 + NBARS2 * 8;
constexpr int OFF_ABORT2 = OFF_TMEM_SLOT2 + 8;
constexpr int OFF_EPI2 = (OFF_ABORT2 + 8 + 15) & ~15;   // per epilogue warp: 32 rows x 64 B
constexpr int EPI_WARP_BYTES = 32 * 64;
constexpr int SMEM2_BYTES = OFF_EPI2 + 4 * EPI_WARP_BYTES + 1024;

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// shared::cluster address of the variable at shared::cta address `a` in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t a, uint32_t rank) {
    uint32_t d;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(rank));
    return d;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on a barrier of either
// CTA of the pair (here always the leader's)
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void* tmap, uint32_t bar_cluster, int c0,
                                                 int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar_cluster), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void mma_f8_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// arrive once on the barrier (shared::cluster address, either CTA) when this thread's earlier
// cta_group::2 MMAs have completed
__device__ __forceinline__ void mma_commit_pair(uint32_t bar_cluster) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster)
                 : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
fp8_gemm_pair_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                     const Fp8GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;     // the same offset in both CTAs
    uint8_t* smem = smem_raw + (base - raw_addr);
    const int warp = warp_id(), lane = lane_id();
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const uint32_t bar0 = base + OFF_BAR2;
    auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_ABORT2);
    const WaitCtl wc{abort_flag, p.wait_budget_ns, p.status};

    const int m_tiles = (p.M + 255) / 256, n_tiles = (p.N + BN - 1) / BN;
    const long long tiles = static_cast<long long>(m_tiles) * n_tiles;
    const int nk = (p.K + BK - 1) / BK;
    const long long pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES2; ++s) {
            mbar_init(bar(F2 + s), 1);
            mbar_init(bar(E2 + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(TF2 + b), 1);
            mbar_init(bar(TE2 + b), 256);
        }
        mbar_init(bar(DR2), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(base + OFF_TMEM_SLOT2),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync_all();                 // both CTAs' barriers and TMEM exist before any remote use
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEM_SLOT2);

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs; bytes counted on the leader's FULL) ----------------
        if (lane == 0) {
            tma_prefetch_desc(&tma_a);
            tma_prefetch_desc(&tma_b);
            int par[STAGES2];
            for (int s = 0; s < STAGES2; ++s) par[s] = -1;
            long long it = 0;
            bool ok = true;
            for (long long t = pair; t < tiles && ok; t += npairs) {
                int mb, nbk;
                tile_of(t, m_tiles, n_tiles, mb, nbk);
                const int m0 = mb * 256 + static_cast<int>(rank) * 128;
                const int nb = nbk * BN + static_cast<int>(rank) * 128;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = static_cast<int>(it % STAGES2);
                    const int use = static_cast<int>((it / STAGES2) & 1);
                    ok = wait_thread(bar(E2 + s), use ^ 1, wc);
                    if (!ok) break;
                    if (leader) mbar_arrive_expect_tx(bar(F2 + s), 2 * STAGE2_BYTES);
                    const uint32_t full = mapa_shared(bar(F2 + s), 0);
                    const uint32_t st = base + s * STAGE2_BYTES;
                    tma_load_2d_pair(st, &tma_a, full, kb * BK, m0);
                    tma_load_2d_pair(st + HALF_BYTES, &tma_b, full, kb * BK, nb);
                    par[s] = use;
                }
            }
            if (!ok && leader)
                for (int s = 0; s < STAGES2; ++s)
                    if (par[s] >= 0) drain_wait(bar(F2 + s), par[s]);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (leader only) ----------------
        if (lane == 0 && leader) {
            const uint32_t idesc = make_idesc(1, 0, 0, 0, 0, 256, BN);
            long long it = 0;
            int tc = 0;
            bool ok = true;
            for (long long t = pair; t < tiles && ok; t += npairs, ++tc) {
                const int b = tc & 1;
                ok = wait_thread(bar(TE2 + b), ((tc >> 1) & 1) ^ 1, wc);
                if (!ok) break;
                tc_fence_after();
                const uint32_t acc = tmem + b * BN;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = static_cast<int>(it % STAGES2);
                    ok = wait_thread(bar(F2 + s), static_cast<int>((it / STAGES2) & 1), wc);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t sa = base + s * STAGE2_BYTES, sb = sa + HALF_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk)
                        mma_f8_ss_pair(acc, sdesc_sw128(sa + kk * 32, 16, 1024), sdesc_sw128(sb + kk * 32, 16, 1024),
                                       idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    mma_commit_pair(bar(E2 + s));                          // both CTAs' stage s is free
                    mma_commit_pair(mapa_shared(bar(E2 + s), 1));
                }
                if (!ok) break;
                mma_commit_pair(bar(TF2 + b));
                mma_commit_pair(mapa_shared(bar(TF2 + b), 1));
            }
            mma_commit_pair(bar(DR2));
            drain_wait(bar(DR2), 0);
        }
    } else {
        // ---------------- epilogue (both CTAs: each its own 128 rows) ----------------
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const float sw = *p.b_scale;
        const uint32_t tempty_leader = mapa_shared(bar(TE2), 0);
        int tc = 0;
        bool ok = true;
        for (long long t = pair; t < tiles && ok; t += npairs, ++tc) {
            int mb, nbk;
            tile_of(t, m_tiles, n_tiles, mb, nbk);
            const int m0 = mb * 256 + static_cast<int>(rank) * 128;
            const int n0 = nbk * BN;
            const int b = tc & 1;
            ok = wait_warp(bar(TF2 + b), (tc >> 1) & 1, wc);
            if (!ok) break;
            tc_fence_after();
            const int m = m0 + r;
            const float sc = m < p.M ? p.a_scales[m] * sw : 0.f;
            // each 32-column chunk goes through the warp's 2 KB of shared memory (row-major,
            // 16-byte pieces swizzled by row / 2) so that every store writes 8 whole 64-byte
            // row segments instead of 32 scattered 16-byte pieces
            uint8_t* wbuf = smem + OFF_EPI2 + (warp - 2) * EPI_WARP_BYTES;
            const int row0 = m0 + (warp & 3) * 32;                 // this warp's 32 rows
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem + b * BN + lane_off + c * 32, v);
                tmem_wait_ld();
                uint32_t pw[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pw[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * sc, __uint_as_float(v[2 * e + 1]) * sc);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4*>(wbuf + lane * 64 + ((q ^ ((lane >> 1) & 3)) * 16)) =
                        make_uint4(pw[4 * q], pw[4 * q + 1], pw[4 * q + 2], pw[4 * q + 3]);
                __syncwarp();
                const int n = n0 + c * 32 + (lane & 3) * 8;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int rr = 8 * k + (lane >> 2);
                    const uint4 val = *reinterpret_cast<const uint4*>(wbuf + rr * 64 + (((lane & 3) ^ ((rr >> 1) & 3)) * 16));
                    const int mm = row0 + rr;
                    if (mm < p.M && n < p.N)
                        *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.y) +
                                                  static_cast<long long>(mm) * p.N + n) = val;
                }
                __syncwarp();
            }
            tc_fence_before();
            mbar_arrive_cluster(tempty_leader + 8u * static_cast<uint32_t>(b));   // leader's TEMPTY[b]
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                 // no CTA leaves while its peer may still signal it
    tc_fence_after();
    if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS)
                                : "memory");
}

int sm_count() {
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

}  // namespace fp8

int launch_fp8_quant_rows(const void* x, void* codes, float* scales, int M, int K, cudaStream_t stream) {
    fp8::fp8_quant_rows_kernel<<<fp8::sm_count() * 8, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<uint8_t*>(codes), scales, M, K);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_fp8_quant_tensor(const void* w, void* codes, float* scale2, long long n, cudaStream_t stream) {
    unsigned int* amax_bits = reinterpret_cast<unsigned int*>(scale2 + 1);
    if (cudaMemsetAsync(amax_bits, 0, sizeof(unsigned int), stream) != cudaSuccess) return -1;
    const int grid = fp8::sm_count() * 8;
    fp8::fp8_absmax_kernel<<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(w), n / 8, amax_bits);
    if (cudaGetLastError() != cudaSuccess) return -1;
    fp8::fp8_quant_tensor_kernel<<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(w),
                                                           static_cast<uint8_t*>(codes), n / 8, amax_bits,
                                                           scale2);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_fp8_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tb_half, const Fp8GemmParams& p,
                    cudaStream_t stream) {
    if (p.M > fp8::BM) {
        // CTA pairs: 256 x 256 tiles, one pair per two SMs
        if (configure_smem(reinterpret_cast<const void*>(fp8::fp8_gemm_pair_kernel), fp8::SMEM2_BYTES) != 0)
            return -1;
        const long long tiles = static_cast<long long>((p.M + 255) / 256) * ((p.N + fp8::BN - 1) / fp8::BN);
        const long long pairs = fp8::sm_count() / 2;
        const int grid = 2 * static_cast<int>(tiles < pairs ? tiles : pairs);
        fp8::fp8_gemm_pair_kernel<<<grid, fp8::NTHREADS, fp8::SMEM2_BYTES, stream>>>(ta, tb_half, p);
        return cudaGetLastError() == cudaSuccess ? 0 : -1;
    }
    if (configure_smem(reinterpret_cast<const void*>(fp8::fp8_gemm_kernel), fp8::SMEM_BYTES) != 0) return -1;
    const long long tiles = static_cast<long long>((p.M + fp8::BM - 1) / fp8::BM) * ((p.N + fp8::BN - 1) / fp8::BN);
    const int grid = static_cast<int>(tiles < fp8::sm_count() ? tiles : fp8::sm_count());
    fp8::fp8_gemm_kernel<<<grid, fp8::NTHREADS, fp8::SMEM_BYTES, stream>>>(ta, tb, p);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace wan
