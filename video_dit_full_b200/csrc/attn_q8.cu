// 8-bit forward of the Wan DiT full self-attention on sm_100a.
//
// The pages' 8-bit FlashAttention ("Wan 2.1 ... paper-podcast summary",
// section "干预与形式化": mixed int8/FP8 with FP32 accumulation across blocks;
// kwkr.cn Wan explainer, section 4.2 "FlashAttention3的8-bit优化"), read as:
// int8 Q and K and e4m3 V with per-(batch, head, 64-token block) absmax scales,
// P quantised to e4m3 as e4m3(448 p), and each 64-key block's P V product taken
// out of the tensor core and added in fp32 with that block's V scale.
//
// Two kernels:
//   q8_quantize   one CTA per (tensor, b, h, 64-token block): absmax, scale,
//                 codes (IEEE division, round to nearest even), written
//                 head-major [B, H, S, 128] into the workspace.
//   q8_attn       one CTA per 128-row Q tile of one (b, h), 128-key K/V tiles:
//                 warp 16 TMA, warp 17 tcgen05 issuer, warps 0-7 softmax (two threads
//                 per row, one 64-key block each, partial maxima swapped through
//                 shared memory), warps 8-15 fp32 accumulation of O (two per row).
//                   S = Q8 K8^T          kind::i8, int32 in TMEM (two buffers)
//                   s = S sQ sK / sqrt(D) * log2(e) per 64-key column block
//                   P8 = e4m3(2^(s - m + log2 448)) -> TMEM (over S)
//                   Ob_a, Ob_b = P8 V8 for the tile's two 64-key blocks (kind::f8f6f4)
//                   O = O * 2^(m_old - m) + Ob_a sV_a + Ob_b sV_b   (fp32, registers)
//                 The 448 of P cancels against l = sum 448 p in the epilogue.
#include <cuda.h>

#include "sm100_ptx.cuh"
#include "wan_attn_internal.h"

namespace wan {
namespace q8 {

constexpr int BLK = 64;          // quantisation block (tokens)
constexpr int HD = 128;

__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// one CTA per (tensor, b*H + h, 64-token block), flattened into blockIdx.x in that order;
// 256 threads: thread = (token row of the block, quarter of D)
__global__ void __launch_bounds__(256) q8_quantize_kernel(const Q8QuantParams p) {
    const long long id = blockIdx.x;
    const int blk = static_cast<int>(id % p.nblk);
    const int bh = static_cast<int>((id / p.nblk) % (static_cast<long long>(p.B) * p.H));
    const int which = static_cast<int>(id / (static_cast<long long>(p.nblk) * p.B * p.H));   // 0 Q, 1 K, 2 V
    const int b = bh / p.H, h = bh % p.H;
    const int row = threadIdx.x >> 2, part = threadIdx.x & 3;
    const int tok = blk * BLK + row;
    const bool valid = tok < p.S;
    const __nv_bfloat16* src = which == 0 ? p.q : which == 1 ? p.k : p.v;
    float x[32];
    if (valid) {
        const uint4* s4 = reinterpret_cast<const uint4*>(
            src + ((static_cast<size_t>(b) * p.S + tok) * p.H + h) * HD + part * 32);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const uint4 w = s4[u];
            const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(b2[e]);
                x[u * 8 + 2 * e] = f.x;
                x[u * 8 + 2 * e + 1] = f.y;
            }
        }
    } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = 0.f;
    }
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    __shared__ float warp_max[8];
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = warp_max[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) amax = fmaxf(amax, warp_max[w]);
    const float qmax = which == 2 ? 448.f : 127.f;
    const float scale = amax > 0.f ? __fdiv_rn(amax, qmax) : 1.f;
    const size_t out_off = ((static_cast<size_t>(bh) * p.S) + tok) * HD + part * 32;
    if (threadIdx.x == 0) {
        float* sc = which == 0 ? p.sq : which == 1 ? p.sk : p.sv;
        sc[static_cast<size_t>(bh) * p.nblk + blk] = scale;
    }
    if (!valid) return;
    uint32_t w[8];
    if (which < 2) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            uint32_t word = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float c = rintf(__fdiv_rn(x[u * 4 + e], scale));
                c = fminf(fmaxf(c, -127.f), 127.f);
                word |= (static_cast<uint32_t>(static_cast<int>(c)) & 0xFFu) << (8 * e);
            }
            w[u] = word;
        }
        int8_t* dst = (which == 0 ? p.q8 : p.k8) + out_off;
        uint4* d4 = reinterpret_cast<uint4*>(dst);
        d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
    } else {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint32_t lo = pack_e4m3x2(__fdiv_rn(x[u * 4], scale), __fdiv_rn(x[u * 4 + 1], scale));
            const uint32_t hi = pack_e4m3x2(__fdiv_rn(x[u * 4 + 2], scale), __fdiv_rn(x[u * 4 + 3], scale));
            w[u] = lo | (hi << 16);
        }
        uint4* d4 = reinterpret_cast<uint4*>(p.v8 + out_off);
        d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
}

constexpr int BM = 128;                     // Q rows per CTA
constexpr int BN = 128;                     // keys per K/V tile (two quantisation blocks)
constexpr int T8 = BM * HD;                 // 16 KB 8-bit tile
constexpr int STAGES = 3;
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + T8;
constexpr int OFF_V = OFF_K + STAGES * T8;
constexpr int OFF_ALPHA = OFF_V + STAGES * T8;        // 4 x 128 fp32 rescale factors
constexpr int OFF_STAT = OFF_ALPHA + 4 * BM * 4;      // final m per row, l per (half, row)
constexpr int OFF_XMAX = OFF_STAT + 3 * BM * 4;       // [parity][half][row] partial row maxima
constexpr int OFF_BAR = OFF_XMAX + 2 * 2 * BM * 4;
enum Bar { Q_FULL = 0, K_FULL = 1, K_EMPTY = 4, V_FULL = 7, V_EMPTY = 10, S_FULL = 13, P_READY = 15,
           ALPHA_READY = 17, OB_FULL = 21, OB_FREE = 22, STATS = 23, DRAIN = 24, XCHG = 25, NBARS = 27 };
constexpr int OFF_TMEM_SLOT = OFF_BAR + NBARS * 8;
constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
constexpr int SMEM_BYTES = OFF_ABORT + 8 + 1024;
// warps 0-7 softmax (two threads per row: warps 0-3 keys 0-63 of a tile = one quantisation
// block, warps 4-7 keys 64-127), warps 8-15 fp32 accumulation of O (two threads per row:
// d 0-63 / 64-127), 16 TMA, 17 MMA
constexpr int NTHREADS = 576;
constexpr int WARP_TMA = 16, WARP_MMA = 17;
constexpr int HALF_THREADS = 256;
#ifndef WAN_Q8_POLY_PAIRS
#define WAN_Q8_POLY_PAIRS 0            // of every 8 pairs of exponentials, this many use exp2_poly3
#endif
constexpr int Q8_POLY_PAIRS = WAN_Q8_POLY_PAIRS;
constexpr uint32_t TMEM_COLS = 512;         // S0 | S1 (int32, P8 over the first 32 columns) | Ob_a | Ob_b
constexpr uint32_t T_OBA = 256, T_OBB = 384;
constexpr float LOG2_448 = 8.807354922057604f;

// S (int32) = Q8 K8^T: both [128 rows][128 bytes] K-major with the 128-byte swizzle, K = 32 per MMA.
__device__ __forceinline__ void issue_qk8(uint32_t d_tmem, uint32_t q_smem, uint32_t k_smem, uint32_t idesc) {
#pragma unroll
    for (int kk = 0; kk < HD / 32; ++kk)
        mma_i8_ss(d_tmem, sdesc_sw128(q_smem + kk * 32, 16, 1024), sdesc_sw128(k_smem + kk * 32, 16, 1024),
                  idesc, kk > 0 ? 1u : 0u);
}

// Ob_a, Ob_b = P8 V8 for keys 0-63 and 64-127 of the tile; P8 in TMEM (4 per column; keys
// 0-63 at columns 0-15, keys 64-127 at columns 64-79, each written by the thread that read them),
// V8 [key][d] MN-major (one 128-byte swizzle atom spans all 128 d), 32 keys per MMA.
__device__ __forceinline__ void issue_pv8(uint32_t tmem, uint32_t p_tmem, uint32_t v_smem, uint32_t idesc) {
#pragma unroll
    for (int a = 0; a < 2; ++a) {
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
            mma_f8_ts(tmem + (a ? T_OBB : T_OBA), p_tmem + a * 64 + kk * 8,
                      sdesc_sw128(v_smem + a * 8192 + kk * 4096, 16, 1024), idesc, kk > 0 ? 1u : 0u);
    }
}

__global__ void __launch_bounds__(NTHREADS, 1)
q8_attn_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
               const __grid_constant__ CUtensorMap tmv, const Q8AttnParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_addr);

    const int warp = warp_id();
    const int lane = lane_id();
    const int h = blockIdx.y, b = blockIdx.z;
    const int bh = b * p.H + h;
    const int q0 = blockIdx.x * BM;
    const int S = p.S;
    const int nkv = (S + BN - 1) / BN;

    const uint32_t sQ = base + OFF_Q, sK = base + OFF_K, sV = base + OFF_V;
    float* alpha_buf = reinterpret_cast<float*>(smem + OFF_ALPHA);
    float* stat_m = reinterpret_cast<float*>(smem + OFF_STAT);
    float* stat_l = stat_m + BM;                           // [half][row]
    const uint32_t bar0 = base + OFF_BAR;
    auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
    const WaitCtl wc{abort_flag, p.wait_budget_ns, p.status};

    if (threadIdx.x == 0) {
        mbar_init(bar(Q_FULL), 1);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar(K_FULL + s), 1);
            mbar_init(bar(K_EMPTY + s), 1);
            mbar_init(bar(V_FULL + s), 1);
            mbar_init(bar(V_EMPTY + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(S_FULL + s), 1);
            mbar_init(bar(P_READY + s), HALF_THREADS);
            mbar_init(bar(XCHG + s), HALF_THREADS);
        }
        for (int s = 0; s < 4; ++s) mbar_init(bar(ALPHA_READY + s), HALF_THREADS);
        mbar_init(bar(OB_FULL), 1);
        mbar_init(bar(OB_FREE), HALF_THREADS);
        mbar_init(bar(STATS), HALF_THREADS);
        mbar_init(bar(DRAIN), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == WARP_MMA) {
        tmem_alloc(base + OFF_TMEM_SLOT, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEM_SLOT);

    if (warp == WARP_TMA) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&tmq);
            tma_prefetch_desc(&tmk);
            tma_prefetch_desc(&tmv);
            mbar_arrive_expect_tx(bar(Q_FULL), T8);
            tma_load_3d(sQ, &tmq, bar(Q_FULL), 0, q0, bh);
            int kpar[STAGES], vpar[STAGES];
            for (int s = 0; s < STAGES; ++s) kpar[s] = vpar[s] = -1;
            bool ok = true;
            for (int j = 0; j < nkv; ++j) {
                const int s = j % STAGES;
                const int use = (j / STAGES) & 1;
                ok = wait_thread(bar(K_EMPTY + s), use ^ 1, wc);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(K_FULL + s), T8);
                tma_load_3d(sK + s * T8, &tmk, bar(K_FULL + s), 0, j * BN, bh);
                kpar[s] = use;
                ok = wait_thread(bar(V_EMPTY + s), use ^ 1, wc);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(V_FULL + s), T8);
                tma_load_3d(sV + s * T8, &tmv, bar(V_FULL + s), 0, j * BN, bh);
                vpar[s] = use;
            }
            if (!ok) {
                drain_wait(bar(Q_FULL), 0);
                for (int s = 0; s < STAGES; ++s) {
                    if (kpar[s] >= 0) drain_wait(bar(K_FULL + s), kpar[s]);
                    if (vpar[s] >= 0) drain_wait(bar(V_FULL + s), vpar[s]);
                }
            }
        }
    } else if (warp == WARP_MMA) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0) {
            const uint32_t idesc_qk = make_idesc(2, 1, 1, 0, 0, BM, BN);   // s32 <- s8 x s8
            const uint32_t idesc_pv = make_idesc(1, 0, 0, 0, 1, BM, HD);   // f32 <- e4m3 x e4m3, V MN-major
            bool ok = wait_thread(bar(Q_FULL), 0, wc);
            for (int j = 0; j < 2 && j < nkv && ok; ++j) {
                ok = wait_thread(bar(K_FULL + j), 0, wc);
                if (!ok) break;
                tc_fence_after();
                issue_qk8(tmem + j * BN, sQ, sK + j * T8, idesc_qk);
                mma_commit(bar(S_FULL + j));
                mma_commit(bar(K_EMPTY + j));
            }
            for (int j = 0; j < nkv && ok; ++j) {
                const int sb = j & 1;
                const int vs = j % STAGES;
                ok = wait_thread(bar(P_READY + sb), (j >> 1) & 1, wc);
                if (ok && j > 0) ok = wait_thread(bar(OB_FREE), (j - 1) & 1, wc);
                if (ok) ok = wait_thread(bar(V_FULL + vs), (j / STAGES) & 1, wc);
                if (!ok) break;
                tc_fence_after();
                issue_pv8(tmem, tmem + sb * BN, sV + vs * T8, idesc_pv);
                mma_commit(bar(OB_FULL));
                mma_commit(bar(V_EMPTY + vs));
                if (j + 2 < nkv) {
                    const int ks = (j + 2) % STAGES;
                    ok = wait_thread(bar(K_FULL + ks), ((j + 2) / STAGES) & 1, wc);
                    if (!ok) break;
                    tc_fence_after();
                    issue_qk8(tmem + sb * BN, sQ, sK + ks * T8, idesc_qk);   // after P V read this buffer
                    mma_commit(bar(S_FULL + sb));
                    mma_commit(bar(K_EMPTY + ks));
                }
            }
            mma_commit(bar(DRAIN));
            drain_wait(bar(DRAIN), 0);
        }
    } else if (warp < 8) {
        // ------------------- softmax (row r, key half hc = one 64-key block) -------
        const int hc = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const int row = q0 + r;
        const float* sk = p.sk + static_cast<size_t>(bh) * p.nblk;
        const float sq_row = p.sq[static_cast<size_t>(bh) * p.nblk + min(row, S - 1) / BLK];
        float* xmax = reinterpret_cast<float*>(smem + OFF_XMAX);
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nkv && ok; ++j) {
            const int sb = j & 1;
            const int kb = 2 * j + hc;                      // this thread's quantisation block
            ok = wait_warp(bar(S_FULL + sb), (j >> 1) & 1, wc);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tS = tmem + sb * BN + lane_off + hc * 64;
            uint32_t sr[64];
            tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
            tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
            tmem_wait_ld();
            const float cs = kb < p.nblk ? sq_row * sk[kb] * p.scale_log2 : 0.f;
            float* s = reinterpret_cast<float*>(sr);
            // int32 -> fp32 without the conversion unit: |S| <= 128*127*127 < 2^22, so
            // adding 1.5*2^23 as a float bit pattern and subtracting it back is exact.
#pragma unroll
            for (int c = 0; c < 64; ++c)
                s[c] = (__int_as_float(static_cast<int>(sr[c]) + 0x4B400000) - 12582912.f) * cs;
            const int valid = S - j * BN - hc * 64;
            if (valid < 64) {
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    if (c >= valid) s[c] = -INFINITY;
            }
            float m8[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) m8[c] = s[c];
#pragma unroll
            for (int c = 8; c < 64; ++c) m8[c & 7] = fmaxf(m8[c & 7], s[c]);
#pragma unroll
            for (int w = 4; w > 0; w >>= 1)
#pragma unroll
                for (int c = 0; c < w; ++c) m8[c] = fmaxf(m8[c], m8[c + w]);
            // swap partial maxima with the other half of the row
            const int xb = (sb * 2) * BM;
            xmax[xb + hc * BM + r] = m8[0];
            mbar_arrive(bar(XCHG + sb));
            ok = wait_warp(bar(XCHG + sb), (j >> 1) & 1, wc);
            if (!ok) break;
            const float mx = fmaxf(m8[0], xmax[xb + (hc ^ 1) * BM + r]);
            const float m_new = fmaxf(m, mx);
            const float alpha = ex2_approx(m - m_new);
            const float bias = m_new - LOG2_448;       // p * 448 = 2^(s - bias) <= 448
            float sum4[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t pk[16];
#pragma unroll
            for (int w = 0; w < 16; ++w) {
                const bool poly = ((2 * w) & 7) < 2 * Q8_POLY_PAIRS;
                const float x0 = s[4 * w] - bias, x1 = s[4 * w + 1] - bias;
                const float x2 = s[4 * w + 2] - bias, x3 = s[4 * w + 3] - bias;
                const float p0 = poly ? exp2_poly3(x0) : ex2_approx(x0);
                const float p1 = poly ? exp2_poly3(x1) : ex2_approx(x1);
                const float p2 = poly ? exp2_poly3(x2) : ex2_approx(x2);
                const float p3 = poly ? exp2_poly3(x3) : ex2_approx(x3);
                sum4[w & 3] += (p0 + p1) + (p2 + p3);
                pk[w] = pack_e4m3x2(p0, p1) | (pack_e4m3x2(p2, p3) << 16);
            }
            tmem_st16(tS, pk);                                 // P8 over the columns this thread read
            l = l * alpha + ((sum4[0] + sum4[1]) + (sum4[2] + sum4[3]));
            m = m_new;
            if (hc == 0) alpha_buf[(j & 3) * BM + r] = alpha;
            mbar_arrive(bar(ALPHA_READY + (j & 3)));
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(P_READY + sb));
        }
        if (ok) {
            if (hc == 0) stat_m[r] = m;
            stat_l[hc * BM + r] = l;
            mbar_arrive(bar(STATS));
        }
    } else {
        // ------------- fp32 accumulation of O (row r, d half hd) -----------------
        const int hd = (warp >> 2) & 1;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const int row = q0 + r;
        const float* sv = p.sv + static_cast<size_t>(bh) * p.nblk;
        float o[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) o[c] = 0.f;
        bool ok = true;
        for (int j = 0; j < nkv && ok; ++j) {
            ok = wait_warp(bar(ALPHA_READY + (j & 3)), (j >> 2) & 1, wc);
            if (!ok) break;
            const float alpha = alpha_buf[(j & 3) * BM + r];
            ok = wait_warp(bar(OB_FULL), j & 1, wc);
            if (!ok) break;
            tc_fence_after();
            const int kb = 2 * j;
            const float sva = sv[kb];
            const float svb = kb + 1 < p.nblk ? sv[kb + 1] : 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t a[16], bb[16];
                tmem_ld16(tmem + T_OBA + lane_off + hd * 64 + q * 16, a);
                tmem_ld16(tmem + T_OBB + lane_off + hd * 64 + q * 16, bb);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    o[q * 16 + e] = fmaf(__uint_as_float(a[e]), sva,
                                         fmaf(__uint_as_float(bb[e]), svb, o[q * 16 + e] * alpha));
            }
            tc_fence_before();
            mbar_arrive(bar(OB_FREE));
        }
        if (ok) ok = wait_warp(bar(STATS), 0, wc);
        if (ok && row < S) {
            const float m = stat_m[r], l = stat_l[r] + stat_l[BM + r];
            const float inv_l = 1.f / l;
            __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) +
                                  ((static_cast<size_t>(b) * S + row) * p.H + h) * HD + hd * 64;
            uint4* d4 = reinterpret_cast<uint4*>(orow);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                d4[u] = make_uint4(pack_bf16x2(o[8 * u] * inv_l, o[8 * u + 1] * inv_l),
                                   pack_bf16x2(o[8 * u + 2] * inv_l, o[8 * u + 3] * inv_l),
                                   pack_bf16x2(o[8 * u + 4] * inv_l, o[8 * u + 5] * inv_l),
                                   pack_bf16x2(o[8 * u + 6] * inv_l, o[8 * u + 7] * inv_l));
            if (hd == 0)
                p.lse[static_cast<size_t>(bh) * S + row] = (m + log2f(l) - LOG2_448) * 0.69314718055994531f;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == WARP_MMA) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace q8

int launch_q8(const Q8QuantParams& qp, const CUtensorMap& tq8, const CUtensorMap& tk8, const CUtensorMap& tv8,
              const Q8AttnParams& p, cudaStream_t stream) {
    const long long nq = 3ll * qp.nblk * qp.B * qp.H;
    q8::q8_quantize_kernel<<<static_cast<unsigned>(nq), 256, 0, stream>>>(qp);
    if (cudaGetLastError() != cudaSuccess) return -1;
    if (configure_smem(reinterpret_cast<const void*>(q8::q8_attn_kernel), q8::SMEM_BYTES) != 0) return -1;
    const dim3 grid((p.S + q8::BM - 1) / q8::BM, p.H, p.B);
    q8::q8_attn_kernel<<<grid, q8::NTHREADS, q8::SMEM_BYTES, stream>>>(tq8, tk8, tv8, p);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace wan
