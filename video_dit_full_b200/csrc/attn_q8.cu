// 8-bit forward of the Wan DiT full self-attention on sm_100a.
//
// The pages' 8-bit FlashAttention ("Wan 2.1 ... paper-podcast summary",
// section "干预与形式化": mixed int8/FP8 with FP32 accumulation across blocks;
// kwkr.cn Wan explainer, section 4.2 "FlashAttention3的8-bit优化"), read as:
// int8 Q and K with per-(batch, head, 64-token block) absmax/127 scales and e4m3 V
// with per-block power-of-two scales (the smallest 2^k >= absmax/448);
// P quantised to e4m3 with each 64-key block's V scale folded in,
// P8 = e4m3(P_SCALE p sV_block / sV_max); every block's P8 V8 product summed by
// the tensor core's fp32 accumulator; O = that sum * sV_max / P_SCALE / l.
//
// Two kernels:
//   q8_quantize   one CTA per (tensor, b, h, 64-token block): absmax, scale,
//                 codes (fp32 products with the block's reciprocal scale, round to
//                 nearest even), written
//                 head-major [B, H, S, 128] into the workspace.
//   q8_attn       one CTA per pair of 128-row Q tiles of one (b, h), sharing
//                 128-key K8/V8 tiles (three-stage TMA rings); the same ping-pong
//                 as the bf16 forward:
//                   S_t = Q8_t K8^T         kind::i8, int32 in TMEM
//                   s = S sQ sK / sqrt(D) * log2(e) per 64-key column block
//                   P8_t = e4m3(2^(s - m + log2(P_SCALE sV_blk / sV_max)))  -> TMEM (over S_t)
//                   O_t += P8_t V8        kind::f8f6f4, fp32 accumulator in TMEM
//                 warp 8 TMA, warp 9 MMA, warps 0-3 / 4-7 softmax of Q tile 0 / 1.
#include <cuda.h>

#include "sm100_ptx.cuh"
#include "wan_attn_internal.h"

namespace wan {
namespace q8 {

constexpr int BLK = 64;          // quantisation block (tokens)
constexpr int HD = 128;


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
    float scale = 1.f, inv = 1.f;                          // codes = x * inv
    if (amax > 0.f) {
        if (which < 2) {
            scale = __fdiv_rn(amax, 127.f);                   // int8: dequantisation scale absmax / 127
            inv = __fdiv_rn(127.f, amax);                     // one division per block, then products
        } else {
            // e4m3: the smallest power of two >= absmax / 448, so that the ratio of any two
            // of a head's V block scales is an exact power of two (it is folded into P)
            // (at least 2^-126, so every scale is a normal float whose exponent field gives k)
            const float q = __fdiv_rn(amax, 448.f);
            int e;
            const float mant = frexpf(q, &e);                 // q = mant * 2^e, mant in [0.5, 1)
            scale = fmaxf((mant == 0.5f) ? q : ldexpf(1.f, e), 0x1p-126f);
            inv = 1.f / scale;                                // exact: scale is a power of two
        }
    }
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
                float c = rintf(__fmul_rn(x[u * 4 + e], inv));
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
            const uint32_t lo = pack_e4m3x2(__fmul_rn(x[u * 4], inv), __fmul_rn(x[u * 4 + 1], inv));
            const uint32_t hi = pack_e4m3x2(__fmul_rn(x[u * 4 + 2], inv), __fmul_rn(x[u * 4 + 3], inv));
            w[u] = lo | (hi << 16);
        }
        uint4* d4 = reinterpret_cast<uint4*>(p.v8 + out_off);
        d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
}

constexpr int BM = 128;                     // query rows per Q tile
constexpr int BN = 128;                     // keys per K/V tile (two quantisation blocks)
constexpr int NQ = 2;                       // Q tiles per CTA (they share every K/V tile)
constexpr int T8 = BM * HD;                 // 16 KB 8-bit tile
constexpr int STAGES = 3;
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + NQ * T8;
constexpr int OFF_V = OFF_K + STAGES * T8;
constexpr int OFF_RED = OFF_V + STAGES * T8;          // 16 floats: per-warp partial maxima of sV
constexpr int OFF_BAR = OFF_RED + 64;
enum Bar { Q_FULL = 0, K_FULL = 2, K_EMPTY = 5, V_FULL = 8, V_EMPTY = 11, S_FULL = 14, P_FULL = 16,
           O_FINAL = 18, DRAIN = 20, NBARS = 21 };
constexpr int OFF_TMEM_SLOT = OFF_BAR + NBARS * 8;
constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
constexpr int SMEM_BYTES = OFF_ABORT + 8 + 1024;
constexpr int NTHREADS = 320;               // warps 0-3 softmax of Q tile 0, 4-7 of Q tile 1, 8 TMA, 9 MMA
constexpr uint32_t TMEM_COLS = 512;         // S0 | S1 (int32; P8 over their first 32 columns) | O0 | O1
constexpr uint32_t T_O = 256;
// The running max is moved only when it rises by more than 1 (log2 units), so p <= 2 against
// the max in use; P is then quantised as e4m3(P_SCALE * p * sV_block / sV_max) <= 448.
constexpr float RESCALE_THRESHOLD = 1.0f;
constexpr float P_SCALE = 224.f;
constexpr float LOG2_P_SCALE = 7.807354922057604f;

// S (int32) = Q8 K8^T: both [128 rows][128 bytes] K-major with the 128-byte swizzle, K = 32 per MMA.
__device__ __forceinline__ void issue_qk8(uint32_t d_tmem, uint32_t q_smem, uint32_t k_smem, uint32_t idesc) {
#pragma unroll
    for (int kk = 0; kk < HD / 32; ++kk)
        mma_i8_ss(d_tmem, sdesc_sw128(q_smem + kk * 32, 16, 1024), sdesc_sw128(k_smem + kk * 32, 16, 1024),
                  idesc, kk > 0 ? 1u : 0u);
}

// O (fp32, TMEM) += P8 V8: P8 in TMEM (4 e4m3 per column, columns 0-31), V8 [key][d] MN-major
// (one 128-byte swizzle atom spans all 128 d), 32 keys per MMA.  The tensor core's fp32
// accumulator carries the sum across every 64-key block; each block's V scale is already in P8.
__device__ __forceinline__ void issue_pv8(uint32_t d_tmem, uint32_t p_tmem, uint32_t v_smem, uint32_t idesc,
                                          bool accumulate) {
#pragma unroll
    for (int kk = 0; kk < BN / 32; ++kk)
        mma_f8_ts(d_tmem, p_tmem + kk * 8, sdesc_sw128(v_smem + kk * 4096, 16, 1024), idesc,
                  (accumulate || kk > 0) ? 1u : 0u);
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
    const int q0 = blockIdx.x * (NQ * BM);
    const int S = p.S;
    const int nq = (q0 + BM < S) ? 2 : 1;
    const int nkv = (S + BN - 1) / BN;

    const uint32_t sQ = base + OFF_Q, sK = base + OFF_K, sV = base + OFF_V;
    float* red = reinterpret_cast<float*>(smem + OFF_RED);
    const uint32_t bar0 = base + OFF_BAR;
    auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
    const WaitCtl wc{abort_flag, p.wait_budget_ns, p.status};

    // sV_max of this (b, h): every thread folds a strided share, warps reduce by shuffle
    const float* sv = p.sv + static_cast<size_t>(bh) * p.nblk;
    {
        float mv = 0.f;
        for (int i = threadIdx.x; i < p.nblk; i += NTHREADS) mv = fmaxf(mv, sv[i]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mv = fmaxf(mv, __shfl_xor_sync(0xffffffffu, mv, off));
        if (lane == 0) red[warp] = mv;
    }
    if (threadIdx.x == 0) {
        mbar_init(bar(Q_FULL), 1);
        mbar_init(bar(Q_FULL + 1), 1);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar(K_FULL + s), 1);
            mbar_init(bar(K_EMPTY + s), 1);
            mbar_init(bar(V_FULL + s), 1);
            mbar_init(bar(V_EMPTY + s), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar(S_FULL + t), 1);
            mbar_init(bar(P_FULL + t), BM);
            mbar_init(bar(O_FINAL + t), 1);
        }
        mbar_init(bar(DRAIN), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 9) {
        tmem_alloc(base + OFF_TMEM_SLOT, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEM_SLOT);
    float sv_max = red[0];
#pragma unroll
    for (int w = 1; w < NTHREADS / 32; ++w) sv_max = fmaxf(sv_max, red[w]);

    if (warp == 8) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&tmq);
            tma_prefetch_desc(&tmk);
            tma_prefetch_desc(&tmv);
            for (int t = 0; t < nq; ++t) {
                mbar_arrive_expect_tx(bar(Q_FULL + t), T8);
                tma_load_3d(sQ + t * T8, &tmq, bar(Q_FULL + t), 0, q0 + t * BM, bh);
            }
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
                for (int t = 0; t < nq; ++t) drain_wait(bar(Q_FULL + t), 0);
                for (int s = 0; s < STAGES; ++s) {
                    if (kpar[s] >= 0) drain_wait(bar(K_FULL + s), kpar[s]);
                    if (vpar[s] >= 0) drain_wait(bar(V_FULL + s), vpar[s]);
                }
            }
        }
    } else if (warp == 9) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0) {
            const uint32_t idesc_qk = make_idesc(2, 1, 1, 0, 0, BM, BN);   // s32 <- s8 x s8
            const uint32_t idesc_pv = make_idesc(1, 0, 0, 0, 1, BM, HD);   // f32 <- e4m3 x e4m3, V MN-major
            bool ok = true;
            for (int t = 0; t < nq && ok; ++t) ok = wait_thread(bar(Q_FULL + t), 0, wc);
            if (ok) ok = wait_thread(bar(K_FULL + 0), 0, wc);
            if (ok) {
                tc_fence_after();
                for (int t = 0; t < nq; ++t) {
                    issue_qk8(tmem + t * BN, sQ + t * T8, sK, idesc_qk);
                    mma_commit(bar(S_FULL + t));
                }
                mma_commit(bar(K_EMPTY + 0));
            }
            for (int j = 0; j < nkv && ok; ++j) {
                const int s = j % STAGES;
                const int s1 = (j + 1) % STAGES;
                ok = wait_thread(bar(V_FULL + s), (j / STAGES) & 1, wc);
                for (int t = 0; t < nq && ok; ++t) {
                    ok = wait_thread(bar(P_FULL + t), j & 1, wc);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv8(tmem + T_O + t * HD, tmem + t * BN, sV + s * T8, idesc_pv, j > 0);
                    if (j + 1 == nkv) mma_commit(bar(O_FINAL + t));
                    if (j + 1 < nkv) {
                        if (t == 0) {
                            ok = wait_thread(bar(K_FULL + s1), ((j + 1) / STAGES) & 1, wc);
                            if (!ok) break;
                            tc_fence_after();
                        }
                        issue_qk8(tmem + t * BN, sQ + t * T8, sK + s1 * T8, idesc_qk);   // after P V read it
                        mma_commit(bar(S_FULL + t));
                    }
                }
                if (!ok) break;
                mma_commit(bar(V_EMPTY + s));
                if (j + 1 < nkv) mma_commit(bar(K_EMPTY + s1));
            }
            mma_commit(bar(DRAIN));
            drain_wait(bar(DRAIN), 0);
        }
    } else {
        // ---------------- softmax, O rescale and epilogue (row r of Q tile t) ------------
        const int t = warp >> 2;
        const int r = threadIdx.x & 127;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + t * BN + lane_off;
        const uint32_t tO = tmem + T_O + t * HD + lane_off;
        const int row = q0 + t * BM + r;
        const float* sk = p.sk + static_cast<size_t>(bh) * p.nblk;
        const float sq_row = p.sq[static_cast<size_t>(bh) * p.nblk + min(row, S - 1) / BLK];
        const int sv_max_exp = static_cast<int>(__float_as_uint(sv_max) >> 23);   // positive, normal
        float m_ref = -INFINITY, l = 0.f;
        bool ok = (t < nq);
        for (int j = 0; j < nkv && ok; ++j) {
            ok = wait_warp(bar(S_FULL + t), j & 1, wc);
            if (!ok) break;
            tc_fence_after();
            uint32_t sr[128];
#pragma unroll
            for (int q = 0; q < 4; ++q) tmem_ld32(tS + q * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[q * 32]));
            tmem_wait_ld();
            const int kb = 2 * j;
            const bool has_b = kb + 1 < p.nblk;
            const float ca = sq_row * sk[kb] * p.scale_log2;
            const float cb = has_b ? sq_row * sk[kb + 1] * p.scale_log2 : 0.f;
            float* s = reinterpret_cast<float*>(sr);
            // int32 -> fp32 without the conversion unit: |S| <= 128*127*127 < 2^22, so adding
            // 1.5*2^23 as a float bit pattern and subtracting it back is exact.  Pairs of scores
            // go through packed fp32 instructions (FADD2 / FMUL2).
            {
                const float2 k2 = make_float2(-12582912.f, -12582912.f);
                const float2 ca2 = make_float2(ca, ca), cb2 = make_float2(cb, cb);
#pragma unroll
                for (int c = 0; c < 128; c += 2) {
                    const float2 xm = make_float2(__int_as_float(static_cast<int>(sr[c]) + 0x4B400000),
                                                  __int_as_float(static_cast<int>(sr[c + 1]) + 0x4B400000));
                    const float2 v = fmul2(fadd2(xm, k2), c < 64 ? ca2 : cb2);
                    s[c] = v.x;
                    s[c + 1] = v.y;
                }
            }
            const int valid = S - j * BN;
            if (valid < BN) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c >= valid) s[c] = -INFINITY;
            }
            // row max: 8 chains of three-input maxima, then a short tree
            float m8[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) m8[q] = fmax3(s[q], s[q + 8], s[q + 16]);
#pragma unroll
            for (int q = 24; q < 128; q += 16)
#pragma unroll
                for (int e = 0; e < 8; ++e) m8[e] = (q + 8 + e < 128) ? fmax3(m8[e], s[q + e], s[q + 8 + e])
                                                                       : fmaxf(m8[e], s[q + e]);
            m8[0] = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
            float alpha = 1.f;
            bool moved = false;
            if (m8[0] > m_ref + RESCALE_THRESHOLD) {
                alpha = ex2_approx(m_ref - m8[0]);
                m_ref = m8[0];
                moved = true;
            }
            // P_SCALE * p * sV_blk / sV_max = 2^(s - m_ref + lg_blk), lg_blk = log2(P_SCALE * sV_blk / sV_max)
            // V block scales are normal powers of two: r = sV_blk / sV_max = 2^-k exactly, k read off
            // the exponent fields
            // (k is clamped to 64: any block 2^-20 below the largest already quantises to zero)
            const int ka = min(sv_max_exp - static_cast<int>(__float_as_uint(sv[kb]) >> 23), 64);
            const int kbb = has_b ? min(sv_max_exp - static_cast<int>(__float_as_uint(sv[kb + 1]) >> 23), 64) : 0;
            const float inv_a = __uint_as_float(static_cast<uint32_t>(127 + ka) << 23) * (1.f / P_SCALE);
            const float inv_b = __uint_as_float(static_cast<uint32_t>(127 + kbb) << 23) * (1.f / P_SCALE);
            const float ba = m_ref - (LOG2_P_SCALE - static_cast<float>(ka));
            const float bbias = m_ref - (LOG2_P_SCALE - static_cast<float>(kbb));
            float2 sa2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            float2 sb2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            const float2 nba = make_float2(-ba, -ba), nbb = make_float2(-bbias, -bbias);
            uint32_t pk[32];
#pragma unroll
            for (int w = 0; w < 32; ++w) {
                const float2 nb = w < 16 ? nba : nbb;
                const float2 x01 = fadd2(make_float2(s[4 * w], s[4 * w + 1]), nb);
                const float2 x23 = fadd2(make_float2(s[4 * w + 2], s[4 * w + 3]), nb);
                const float2 p01 = make_float2(ex2_approx(x01.x), ex2_approx(x01.y));
                const float2 p23 = make_float2(ex2_approx(x23.x), ex2_approx(x23.y));
                if (w < 16) sa2[w & 1] = fadd2(sa2[w & 1], fadd2(p01, p23));
                else sb2[w & 1] = fadd2(sb2[w & 1], fadd2(p01, p23));
                pk[w] = pack_e4m3x2(p01.x, p01.y) | (pack_e4m3x2(p23.x, p23.y) << 16);
            }
            tmem_st32(tS, pk);                                   // P8 over S's first 32 columns
            // the row sum counts p itself: scale each block's sum by 1 / (P_SCALE * r_blk) = 2^k / P_SCALE
            const float sum = ((sa2[0].x + sa2[0].y) + (sa2[1].x + sa2[1].y)) * inv_a +
                              ((sb2[0].x + sb2[0].y) + (sb2[1].x + sb2[1].y)) * inv_b;
            l = l * alpha + sum;
            if (j > 0 && __any_sync(0xffffffffu, moved)) {
#pragma unroll 1
                for (int q = 0; q < 4; ++q) {
                    uint32_t o[32];
                    tmem_ld32(tO + q * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(tO + q * 32, o);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(P_FULL + t));
        }
        if (ok) ok = wait_warp(bar(O_FINAL + t), 0, wc);
        if (ok) {
            tc_fence_after();
            // O = (sum over blocks of P8 V8) * sV_max / P_SCALE / l
            const float mul = sv_max / (P_SCALE * l);
            __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) +
                                  ((static_cast<size_t>(b) * S + row) * p.H + h) * HD;
#pragma unroll 1
            for (int q = 0; q < 4; ++q) {
                uint32_t o[32];
                tmem_ld32(tO + q * 32, o);
                tmem_wait_ld();
                uint4 pk4[4];
                uint32_t* pw = reinterpret_cast<uint32_t*>(pk4);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pw[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * mul, __uint_as_float(o[2 * e + 1]) * mul);
                if (row < S) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[e] = pk4[e];
                }
            }
            if (row < S) p.lse[static_cast<size_t>(bh) * S + row] = (m_ref + log2f(l)) * 0.69314718055994531f;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace q8

int launch_q8(const Q8QuantParams& qp, const CUtensorMap& tq8, const CUtensorMap& tk8, const CUtensorMap& tv8,
              const Q8AttnParams& p, cudaStream_t stream) {
    const long long nq = 3ll * qp.nblk * qp.B * qp.H;
    q8::q8_quantize_kernel<<<static_cast<unsigned>(nq), 256, 0, stream>>>(qp);
    if (cudaGetLastError() != cudaSuccess) return -1;
    if (configure_smem(reinterpret_cast<const void*>(q8::q8_attn_kernel), q8::SMEM_BYTES) != 0) return -1;
    const dim3 grid((p.S + q8::NQ * q8::BM - 1) / (q8::NQ * q8::BM), p.H, p.B);
    q8::q8_attn_kernel<<<grid, q8::NTHREADS, q8::SMEM_BYTES, stream>>>(tq8, tk8, tv8, p);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace wan
