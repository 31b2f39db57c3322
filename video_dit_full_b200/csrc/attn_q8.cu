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
//                 64-key K8/V8 tiles (six-stage TMA rings), one quantisation block
//                 per step, S double-buffered in TMEM per Q tile:
//                   S_t = Q8_t K8^T         kind::i8, int32 in TMEM
//                   s = S sQ sK / sqrt(D) * log2(e) per 64-key column block
//                   P8_t = e4m3(2^(s - m + log2(P_SCALE sV_blk / sV_max)))  -> TMEM (over S_t)
//                   O_t += P8_t V8        kind::f8f6f4, fp32 accumulator in TMEM
//                 warp 8 TMA, warps 9 / 10 MMA, warps 0-3 / 4-7 softmax of Q tile 0 / 1.
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
constexpr int BN = 64;                      // keys per step: one quantisation block
constexpr int NQ = 2;                       // Q tiles per CTA (they share every K/V tile)
constexpr int TQ8 = BM * HD;                // 16 KB 8-bit Q tile
constexpr int TKV8 = BN * HD;               // 8 KB 8-bit K or V tile
constexpr int STAGES = 6;
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + NQ * TQ8;
constexpr int OFF_V = OFF_K + STAGES * TKV8;
constexpr int OFF_RED = OFF_V + STAGES * TKV8;        // 16 floats: per-warp partial maxima of sV
constexpr int OFF_BAR = OFF_RED + 64;
// KV_FULL + s / KV_EMPTY + s: K and V of one 64-key block, loaded and released together;
// S_FULL + 2 t + b: S of Q tile t in buffer b is ready; P_FULL + 2 t + b: P of tile t in buffer
// b is; PV_LAST + t: P V of the next-to-last block has landed in O; O_FINAL + t: the last has.
// Per-buffer barriers keep each waiter at most one phase behind its barrier: the softmax may
// finish steps j and j + 1 before the MMA takes P of step j, but not step j + 2 (its S is
// computed only after that), so a parity names the phase without ambiguity.
enum Bar { Q_FULL = 0, KV_FULL = 2, KV_EMPTY = KV_FULL + STAGES, S_FULL = KV_EMPTY + STAGES,
           P_FULL = S_FULL + 4, PV_LAST = P_FULL + 4, O_FINAL = PV_LAST + 2, DRAIN = O_FINAL + 2,
           NBARS = DRAIN + 2 };
constexpr int OFF_TMEM_SLOT = OFF_BAR + NBARS * 8;
constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
constexpr int SMEM_BYTES = OFF_ABORT + 8 + 1024;
// warps 0-3 softmax of Q tile 0, 4-7 of Q tile 1, 8 TMA, 9 and 10 the MMAs of Q tile 0 and 1: one
// issuing thread per tile, so that the two tiles' MMA chains do not queue behind each other
constexpr int NTHREADS = 352;
// TMEM: S of tile t, buffer b (int32, 64 columns; P8 over its first 16) at 64 (2 t + b); O of
// tile t (fp32, 128 columns) at 256 + 128 t.  With S double-buffered, the MMA computes the next
// S of a tile while its softmax works on this one.
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t T_O = 256;
// The running max is moved only when it rises by more than 1 (log2 units), so p <= 2 against
// the max in use; P is then quantised as e4m3(P_SCALE * p * sV_block / sV_max) <= 448.
constexpr float RESCALE_THRESHOLD = 1.0f;
#ifndef WAN_Q8_POLY_GROUPS
#define WAN_Q8_POLY_GROUPS 3        // of every 8 groups of 4 exponentials in P, this many use exp2_poly2_x2
#endif
constexpr int Q8_POLY_GROUPS = WAN_Q8_POLY_GROUPS;
constexpr float P_SCALE = 224.f;
constexpr float LOG2_P_SCALE = 7.807354922057604f;

// S (int32) = Q8 K8^T: Q [128 rows][128 bytes], K [64 rows][128 bytes], both K-major with the
// 128-byte swizzle, K = 32 per MMA (mma4_i8_ss).  O (fp32, TMEM) += P8 V8: P8 in TMEM (4 e4m3 per
// column, 16 columns for the 64 keys), V8 [key][d] MN-major (one 128-byte swizzle atom spans all
// 128 d), 32 keys per MMA (mma2_f8_ts).  The tensor core's fp32 accumulator carries the sum
// across every 64-key block; each block's V scale is already in P8.

__global__ void __launch_bounds__(NTHREADS, 1)
q8_attn_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
               const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
               const Q8AttnParams p) {
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
    const int nkv = (S + BN - 1) / BN;             // = the number of 64-token blocks

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
        for (int t = 0; t < NQ; ++t) mbar_init(bar(Q_FULL + t), 1);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar(KV_FULL + s), 1);
            mbar_init(bar(KV_EMPTY + s), nq);         // released by each tile's MMA thread
        }
        for (int i = 0; i < 4; ++i) {
            mbar_init(bar(S_FULL + i), 1);
            mbar_init(bar(P_FULL + i), BM);
        }
        for (int t = 0; t < NQ; ++t) {
            mbar_init(bar(PV_LAST + t), 1);
            mbar_init(bar(O_FINAL + t), 1);
        }
        mbar_init(bar(DRAIN), 1);
        mbar_init(bar(DRAIN + 1), 1);
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
                mbar_arrive_expect_tx(bar(Q_FULL + t), TQ8);
                tma_load_3d(sQ + t * TQ8, &tmq, bar(Q_FULL + t), 0, q0 + t * BM, bh);
            }
            int par[STAGES];
            for (int s = 0; s < STAGES; ++s) par[s] = -1;
            bool ok = true;
            for (int j = 0; j < nkv; ++j) {
                const int s = j % STAGES;
                const int use = (j / STAGES) & 1;
                ok = wait_thread(bar(KV_EMPTY + s), use ^ 1, wc);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(KV_FULL + s), 2 * TKV8);
                tma_load_3d(sK + s * TKV8, &tmk, bar(KV_FULL + s), 0, j * BN, bh);
                tma_load_3d(sV + s * TKV8, &tmv, bar(KV_FULL + s), 0, j * BN, bh);
                par[s] = use;
            }
            if (!ok) {
                for (int t = 0; t < nq; ++t) drain_wait(bar(Q_FULL + t), 0);
                for (int s = 0; s < STAGES; ++s)
                    if (par[s] >= 0) drain_wait(bar(KV_FULL + s), par[s]);
            }
        }
    } else if (warp >= 9) {
        // ----------------------- MMA issuer of Q tile t = warp - 9 ------------------------
        // S(t, j) goes to buffer j % 2.  S of the first two steps is computed up front; after
        // P(t, j) V(j) the MMA issues S(t, j + 2) into the buffer P(t, j) has just been read
        // from (the tensor core executes one thread's MMAs in order).
        const int t = warp - 9;
        if (lane == 0 && t < nq) {
            const uint32_t idesc_qk = make_idesc(2, 1, 1, 0, 0, BM, BN);   // s32 <- s8 x s8
            const uint32_t idesc_pv = make_idesc(1, 0, 0, 0, 1, BM, HD);   // f32 <- e4m3 x e4m3, V MN-major
            const uint32_t to = tmem + T_O + t * HD;
            auto sbuf = [&](int j) { return tmem + static_cast<uint32_t>((2 * t + (j & 1)) * BN); };
            // descriptor halves built once: Q of this tile, K and V of stage 0 (a stage is TKV8 / 16
            // address units further on); one common high half
            const uint32_t hi = sdesc_hi();
            const uint32_t q_lo = sdesc_lo(sQ + t * TQ8, 16), k_lo = sdesc_lo(sK, 16), v_lo = sdesc_lo(sV, 16);
            auto issue_qk8 = [&](int j, int st) { mma4_i8_ss(sbuf(j), q_lo, k_lo + st * (TKV8 / 16), hi, idesc_qk); };
            auto issue_pv8 = [&](int j, int st) {
                mma2_f8_ts(to, sbuf(j), v_lo + st * (TKV8 / 16), hi, idesc_pv, j > 0 ? 1u : 0u);
            };
            bool ok = wait_thread(bar(Q_FULL + t), 0, wc);
            for (int j = 0; j < 2 && j < nkv && ok; ++j) {
                ok = wait_thread(bar(KV_FULL + j), 0, wc);
                if (!ok) break;
                tc_fence_after();
                issue_qk8(j, j);
                mma_commit(bar(S_FULL + 2 * t + j));
            }
            for (int j = 0; j < nkv && ok; ++j) {
                const int s = j % STAGES;
                const int j2 = j + 2, s2 = j2 % STAGES;
                const bool next = j2 < nkv;
                // K and V of block j arrived together (K's wait was two steps ago)
                if (next) ok = wait_thread(bar(KV_FULL + s2), (j2 / STAGES) & 1, wc);
                if (ok) ok = wait_thread(bar(P_FULL + 2 * t + (j & 1)), (j >> 1) & 1, wc);
                if (!ok) break;
                tc_fence_after();
                issue_pv8(j, s);
                mma_commit(bar(KV_EMPTY + s));               // after K(j)'s and V(j)'s last readers
                if (j + 2 == nkv) mma_commit(bar(PV_LAST + t));
                if (j + 1 == nkv) mma_commit(bar(O_FINAL + t));
                if (next) {
                    issue_qk8(j, s2);
                    mma_commit(bar(S_FULL + 2 * t + (j & 1)));
                }
            }
            mma_commit(bar(DRAIN + t));
            drain_wait(bar(DRAIN + t), 0);
        }
    } else {
        // ---------------- softmax, O rescale and epilogue (row r of Q tile t) ------------
        const int t = warp >> 2;
        const int r = threadIdx.x & 127;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tO = tmem + T_O + t * HD + lane_off;
        const int row = q0 + t * BM + r;
        const float* sk = p.sk + static_cast<size_t>(bh) * p.nblk;
        const float sq_row = p.sq[static_cast<size_t>(bh) * p.nblk + min(row, S - 1) / BLK];
        const int sv_max_exp = static_cast<int>(__float_as_uint(sv_max) >> 23);   // positive, normal
        float m_ref = -INFINITY, l = 0.f;
        bool ok = (t < nq);
        // the step's K and V block scales, loaded one step ahead
        float sk_cur = sk[0], sv_cur = sv[0];
        for (int j = 0; j < nkv && ok; ++j) {
            const float sk_next = j + 1 < nkv ? sk[j + 1] : 0.f;
            const float sv_next = j + 1 < nkv ? sv[j + 1] : 0.f;
            ok = wait_warp(bar(S_FULL + 2 * t + (j & 1)), (j >> 1) & 1, wc);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tS = tmem + static_cast<uint32_t>((2 * t + (j & 1)) * BN) + lane_off;
            const int valid = S - j * BN;                    // keys of this block that exist
            // c > 0 even for an all-zero block, so that -inf * c stays -inf below
            const float c = fmaxf(sq_row * sk_cur * p.scale_log2, 1e-30f);
            // P_SCALE * p * sV_blk / sV_max = 2^(s - m_ref + lg_blk), lg_blk = log2(P_SCALE * sV_blk / sV_max)
            // V block scales are normal powers of two: r = sV_blk / sV_max = 2^-k exactly, k read off
            // the exponent fields
            // (k is clamped to 64: any block 2^-20 below the largest already quantises to zero)
            const int kx = min(sv_max_exp - static_cast<int>(__float_as_uint(sv_cur) >> 23), 64);
            const float inv = __uint_as_float(static_cast<uint32_t>(127 + kx) << 23) * (1.f / P_SCALE);
            const float2 c2 = make_float2(c, c);
            // S: the int32 sums convert to fp32 exactly (|S| <= 128*127*127 < 2^24), keys past S
            // masked; the block's max
            uint32_t sr[64];
            float* xm = reinterpret_cast<float*>(sr);     // S as fp32, in place
            tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
            tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 64; ++e) xm[e] = __int2float_rn(static_cast<int>(sr[e]));
            if (valid < BN) {
#pragma unroll
                for (int e = 0; e < 64; ++e)
                    if (e >= valid) xm[e] = -INFINITY;
            }
            float m4[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) m4[q] = fmax3(xm[q], xm[q + 4], xm[q + 8]);
#pragma unroll
            for (int e = 12; e + 8 <= 64; e += 8)
#pragma unroll
                for (int q = 0; q < 4; ++q) m4[q] = fmax3(m4[q], xm[e + q], xm[e + 4 + q]);
#pragma unroll
            for (int q = 0; q < 4; ++q) m4[q] = fmaxf(m4[q], xm[60 + q]);
            const float mx = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3])) * c;
            float alpha = 1.f;
            bool moved = false;
            if (mx > m_ref + RESCALE_THRESHOLD) {
                alpha = ex2_approx(m_ref - mx);
                m_ref = mx;
                moved = true;
            }
            const bool any_moved = __any_sync(0xffffffffu, moved);
            // P8 and the row sum: s - bias = S c - bias in one fused multiply-add per pair
            const float nb = -(m_ref - (LOG2_P_SCALE - static_cast<float>(kx)));
            const float2 n2 = make_float2(nb, nb);
            float2 sum2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            uint32_t pk[16];
#pragma unroll
            for (int w = 0; w < 16; ++w) {
                const float2 x01 = ffma2(make_float2(xm[4 * w], xm[4 * w + 1]), c2, n2);
                const float2 x23 = ffma2(make_float2(xm[4 * w + 2], xm[4 * w + 3]), c2, n2);
                float2 p01, p23;
                if ((w & 7) < Q8_POLY_GROUPS) {
                    p01 = exp2_poly2_x2(x01);
                    p23 = exp2_poly2_x2(x23);
                } else {
                    p01 = make_float2(ex2_approx(x01.x), ex2_approx(x01.y));
                    p23 = make_float2(ex2_approx(x23.x), ex2_approx(x23.y));
                }
                sum2[w & 1] = fadd2(sum2[w & 1], fadd2(p01, p23));
                pk[w] = pack_e4m3x2(p01.x, p01.y) | (pack_e4m3x2(p23.x, p23.y) << 16);
            }
            const float sum = (sum2[0].x + sum2[0].y) + (sum2[1].x + sum2[1].y);
            tmem_st16(tS, pk);                                   // P8 over S's first 16 columns
            // the row sum counts p itself: scale by 1 / (P_SCALE * r_blk) = 2^k / P_SCALE
            l = l * alpha + sum * inv;
            if (j > 0 && any_moved) {
                // O must hold P(j - 1) V(j - 1) before it is rescaled.  S(t, j + 1) is computed
                // after that product (the tile's MMAs run in order), so its barrier says so; the
                // last block, which has no S(t, j + 1), has PV_LAST.
                ok = (j + 1 < nkv) ? wait_warp(bar(S_FULL + 2 * t + ((j + 1) & 1)), ((j + 1) >> 1) & 1, wc)
                                   : wait_warp(bar(PV_LAST + t), 0, wc);
                if (!ok) break;
                tc_fence_after();
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
            mbar_arrive(bar(P_FULL + 2 * t + (j & 1)));
            sk_cur = sk_next;
            sv_cur = sv_next;
        }
        if (ok) ok = wait_warp(bar(O_FINAL + t), 0, wc);
        // O goes out through the K/V ring, free once both tiles' last P V have completed (every
        // block was consumed by both tiles' MMAs and nothing more is loaded): tile t's bf16 O in
        // the ring's 32 KB half t, each thread writing its row in the tensor map's 128-byte-swizzled
        // layout, then one thread stores the tile with two TMA stores (rows past S are not written).
        if (ok && 1 - t < nq) ok = wait_warp(bar(O_FINAL + 1 - t), 0, wc);
        const uint32_t stage = sK + static_cast<uint32_t>(t) * (2 * TQ8);
        if (ok) {
            tc_fence_after();
            // O = (sum over blocks of P8 V8) * sV_max / P_SCALE / l
            const float mul = sv_max / (P_SCALE * l);
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t o[64];
                tmem_ld32(tO + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
                tmem_ld32(tO + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
                tmem_wait_ld();
                uint32_t w[32];
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * mul, __uint_as_float(o[2 * e + 1]) * mul);
                st_row_sw128(stage + half * TQ8, r, w);
            }
            fence_proxy_async_smem();
            if (row < S) p.lse[static_cast<size_t>(bh) * S + row] = (m_ref + log2f(l)) * 0.69314718055994531f;
        }
        named_bar_sync(1 + t, BM);                // every warp of the group, whatever its state
        if (r == 0 && ok && !*abort_flag) {
            tma_store_4d(&tmo, stage, 0, h, q0 + t * BM, b);
            tma_store_4d(&tmo, stage + TQ8, 64, h, q0 + t * BM, b);
            bulk_commit_group();
            bulk_wait_read_all();                 // the ring stays valid until the copies have read it
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace q8

int launch_q8(const Q8QuantParams& qp, const CUtensorMap& tq8, const CUtensorMap& tk8, const CUtensorMap& tv8,
              const CUtensorMap& to, const Q8AttnParams& p, cudaStream_t stream) {
    const long long nq = 3ll * qp.nblk * qp.B * qp.H;
    q8::q8_quantize_kernel<<<static_cast<unsigned>(nq), 256, 0, stream>>>(qp);
    if (cudaGetLastError() != cudaSuccess) return -1;
    if (configure_smem(reinterpret_cast<const void*>(q8::q8_attn_kernel), q8::SMEM_BYTES) != 0) return -1;
    const dim3 grid((p.S + q8::NQ * q8::BM - 1) / (q8::NQ * q8::BM), p.H, p.B);
    q8::q8_attn_kernel<<<grid, q8::NTHREADS, q8::SMEM_BYTES, stream>>>(tq8, tk8, tv8, to, p);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace wan
