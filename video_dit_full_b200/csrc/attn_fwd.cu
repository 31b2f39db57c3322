// bf16 forward of the Wan DiT full (non-causal) spatio-temporal self-attention
// on sm_100a: O = softmax(Q K^T / sqrt(D)) V and the natural-log LSE per row.
//
// What is computed: the DiT block's full spatio-temporal self-attention
// ("Wan 2.1 ... paper-podcast summary", section "干预与形式化": full
// spatio-temporal self-attention, neither windowed nor U-ViT; section
// "先看现象": non-causal attention, forward cost term 4*b*s^2*h).  The same kernel
// serves the block's cross-attention from the video tokens to the 512-token umT5
// text embedding (same summary, section "干预与形式化"): queries and keys then
// have different lengths (S and Skv).
//
// How (one CTA = two 128-row Q tiles of one (batch, head)):
//   warp 8      TMA producer: Q tiles once, then K_j / V_j 128-key tiles into a
//               two-stage ring each (128-byte swizzle, zero fill past S).
//   warp 9      tcgen05 issuer: S_t = Q_t K_j^T into TMEM (fp32), then
//               O_t += P_t V_j with P_t read from TMEM (bf16, aliasing S_t).
//   warps 0-3   softmax of Q tile 0, warps 4-7 of Q tile 1: one row per thread,
//               online max / sum in fp32 with exp2, the running max only moved
//               when it rises by more than 2^8 (O rescaled in TMEM then), P
//               written back to TMEM as bf16; epilogue O / l -> bf16 through the
//               tile's Q buffer and two TMA stores, LSE.
// The two Q tiles ping-pong: while one softmax group works on its S, the
// tensor core runs the other tile's P V and Q K^T.
#include <cuda.h>

#include "sm100_ptx.cuh"
#include "wan_attn_internal.h"

namespace wan {
namespace fwd {

constexpr int BM = 128;        // query rows per Q tile
constexpr int BN = 128;        // keys per K/V tile
constexpr int HD = 128;        // head dimension
constexpr int NQ = 2;          // Q tiles per CTA
constexpr int TILE_BYTES = BM * HD * 2;
constexpr int HALF_BYTES = TILE_BYTES / 2;    // 64 columns of d (one 128-byte swizzle span)
constexpr int STAGES = 2;

constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + NQ * TILE_BYTES;
constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;
constexpr int OFF_BAR = OFF_V + STAGES * TILE_BYTES;
enum Bar { Q_FULL = 0, K_FULL = 2, K_EMPTY = 4, V_FULL = 6, V_EMPTY = 8, S_FULL = 10, P_FULL = 12,
           O_FINAL = 14, DRAIN = 16, NBARS = 17 };
constexpr int OFF_TMEM_SLOT = OFF_BAR + NBARS * 8;
constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
constexpr int SMEM_USED = OFF_ABORT + 8;
constexpr int SMEM_BYTES = SMEM_USED + 1024;   // slack for 1024-byte alignment of the tiles
constexpr int NTHREADS = 320;
constexpr uint32_t TMEM_COLS = 512;            // S0 S1 O0 O1, 128 columns each
constexpr float RESCALE_THRESHOLD = 8.0f;      // log2 units: keep a stale max while p <= 2^8
#ifndef WAN_FWD_POLY_PAIRS
#define WAN_FWD_POLY_PAIRS 1          // of every 8 pairs of exponentials, this many use exp2_poly3_x2
#endif
constexpr int FWD_POLY_PAIRS = WAN_FWD_POLY_PAIRS;


__global__ void __launch_bounds__(NTHREADS, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo, const FwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_addr);

    const int warp = warp_id();
    const int lane = lane_id();
    const int h = blockIdx.y, b = blockIdx.z;
    const int q0 = blockIdx.x * (NQ * BM);
    const int nq = (q0 + BM < p.S) ? 2 : 1;          // second tile empty on a short tail
    const int nkv = (p.Skv + BN - 1) / BN;

    const uint32_t sQ = base + OFF_Q, sK = base + OFF_K, sV = base + OFF_V;
    const uint32_t bar0 = base + OFF_BAR;
    auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
    const WaitCtl wc{abort_flag, p.wait_budget_ns, p.status};

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar(Q_FULL + t), 1);
            mbar_init(bar(K_FULL + t), 1);
            mbar_init(bar(K_EMPTY + t), 1);
            mbar_init(bar(V_FULL + t), 1);
            mbar_init(bar(V_EMPTY + t), 1);
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

    if (warp == 8) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&tmq);
            tma_prefetch_desc(&tmk);
            tma_prefetch_desc(&tmv);
            const uint64_t keep = l2_policy_evict_last();
            for (int t = 0; t < nq; ++t) {
                mbar_arrive_expect_tx(bar(Q_FULL + t), TILE_BYTES);
                tma_load_4d(sQ + t * TILE_BYTES, &tmq, bar(Q_FULL + t), 0, h, q0 + t * BM, b);
                tma_load_4d(sQ + t * TILE_BYTES + HALF_BYTES, &tmq, bar(Q_FULL + t), 64, h, q0 + t * BM, b);
            }
            int kpar[2] = {-1, -1}, vpar[2] = {-1, -1};   // parity of the last copy issued per stage
            bool ok = true;
            for (int j = 0; j < nkv && ok; ++j) {
                const int s = j & 1;
                const int use = (j >> 1) & 1;
                ok = wait_thread(bar(K_EMPTY + s), use ^ 1, wc);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(K_FULL + s), TILE_BYTES);
                tma_load_4d_hint(sK + s * TILE_BYTES, &tmk, bar(K_FULL + s), 0, h, j * BN, b, keep);
                tma_load_4d_hint(sK + s * TILE_BYTES + HALF_BYTES, &tmk, bar(K_FULL + s), 64, h, j * BN, b, keep);
                kpar[s] = use;
                ok = wait_thread(bar(V_EMPTY + s), use ^ 1, wc);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(V_FULL + s), TILE_BYTES);
                tma_load_4d_hint(sV + s * TILE_BYTES, &tmv, bar(V_FULL + s), 0, h, j * BN, b, keep);
                tma_load_4d_hint(sV + s * TILE_BYTES + HALF_BYTES, &tmv, bar(V_FULL + s), 64, h, j * BN, b, keep);
                vpar[s] = use;
            }
            if (!ok) {
                // let the copies already issued land before the CTA's shared memory goes away
                for (int t = 0; t < nq; ++t) drain_wait(bar(Q_FULL + t), 0);
                for (int s = 0; s < 2; ++s) {
                    if (kpar[s] >= 0) drain_wait(bar(K_FULL + s), kpar[s]);
                    if (vpar[s] >= 0) drain_wait(bar(V_FULL + s), vpar[s]);
                }
            }
        }
    } else if (warp == 9) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0) {
            const uint32_t idesc_qk = make_idesc(1, 1, 1, 0, 0, BM, BN);
            const uint32_t idesc_pv = make_idesc(1, 1, 1, 0, 1, BM, HD);
            // descriptor halves built once: the low half carries the address (16-byte units) and
            // the leading offset, the high half is common.  Q K^T: 8 steps of K = 16 over the two
            // 64-wide halves of d (Q and K K-major); P V: 8 steps of 16 keys, P from TMEM, V
            // [key][d] MN-major with its halves of d 16 KB apart (LBO).
            const uint32_t hi = sdesc_hi();
            const uint32_t q_lo = sdesc_lo(sQ, 16), k_lo = sdesc_lo(sK, 16), v_lo = sdesc_lo(sV, HALF_BYTES);
            constexpr uint32_t TILE16 = TILE_BYTES >> 4;
            auto issue_qk = [&](int t_, int s_) {
                mma8_f16_ss<HALF_BYTES / 16, 2>(tmem + t_ * BN, q_lo + t_ * TILE16, k_lo + s_ * TILE16, hi, idesc_qk, 0u);
            };
            auto issue_pv = [&](int t_, int s_, bool acc) {
                mma8_f16_ts<32, 512, 128>(tmem + 256 + t_ * HD, tmem + t_ * BN, v_lo + s_ * TILE16, hi, idesc_pv,
                                          acc ? 1u : 0u);
            };
            bool ok = true;
            for (int t = 0; t < nq && ok; ++t) ok = wait_thread(bar(Q_FULL + t), 0, wc);
            if (ok) ok = wait_thread(bar(K_FULL + 0), 0, wc);
            if (ok) {
                tc_fence_after();
                for (int t = 0; t < nq; ++t) {
                    issue_qk(t, 0);
                    mma_commit(bar(S_FULL + t));
                }
                mma_commit(bar(K_EMPTY + 0));
            }
            for (int j = 0; j < nkv && ok; ++j) {
                const int s = j & 1;
                const int s1 = (j + 1) & 1;
                ok = wait_thread(bar(V_FULL + s), (j >> 1) & 1, wc);
                for (int t = 0; t < nq && ok; ++t) {
                    ok = wait_thread(bar(P_FULL + t), j & 1, wc);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(t, s, j > 0);
                    if (j + 1 == nkv) mma_commit(bar(O_FINAL + t));
                    if (j + 1 < nkv) {
                        if (t == 0) {
                            ok = wait_thread(bar(K_FULL + s1), ((j + 1) >> 1) & 1, wc);
                            if (!ok) break;
                            tc_fence_after();
                        }
                        issue_qk(t, s1);
                        mma_commit(bar(S_FULL + t));
                    }
                }
                if (!ok) break;
                mma_commit(bar(V_EMPTY + s));
                if (j + 1 < nkv) mma_commit(bar(K_EMPTY + s1));
            }
            // every MMA issued so far completes before TMEM is released
            mma_commit(bar(DRAIN));
            drain_wait(bar(DRAIN), 0);
        }
    } else {
        // ------------------------- softmax / correction / epilogue ----------------
        const int t = warp >> 2;                 // Q tile of this warpgroup
        const int r = threadIdx.x & 127;         // row within the tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + t * BN + lane_off;
        const uint32_t tO = tmem + 256 + t * HD + lane_off;
        const int row = q0 + t * BM + r;
        const float c = p.scale_log2;
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
            float* s = reinterpret_cast<float*>(sr);
            const int valid = p.Skv - j * BN;    // keys of this tile that exist
            if (valid < BN) {
#pragma unroll
                for (int q = 0; q < 128; ++q)
                    if (q >= valid) s[q] = -INFINITY;
            }
            // row max: 8 chains of three-input maxima, then a short tree
            float m8[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) m8[q] = fmax3(s[q], s[q + 8], s[q + 16]);
#pragma unroll
            for (int q = 24; q < 128; q += 16)
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    m8[e] = (q + 8 + e < 128) ? fmax3(m8[e], s[q + e], s[q + 8 + e]) : fmaxf(m8[e], s[q + e]);
            const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
            const float m_cand = mx * c;
            float alpha = 1.f;
            bool moved = false;
            if (m_cand > m_ref + RESCALE_THRESHOLD) {
                alpha = ex2_approx(m_ref - m_cand);
                m_ref = m_cand;
                moved = true;
            }
            // P = 2^(s c - m) in packed pairs, the row sum in four independent packed accumulators.
            // Of every 8 pairs FWD_POLY_PAIRS come from the degree-3 polynomial on the FMA pipe and
            // the rest from the MUFU (1 by default; more of them slow the MMA issuer, which shares
            // a sub-partition with two softmax warps, by more than they save).
            const float2 c2 = make_float2(c, c), n2 = make_float2(-m_ref, -m_ref);
            float2 acc[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) acc[a] = make_float2(0.f, 0.f);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t pk[32];
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    const float2 x = ffma2(make_float2(s[half * 64 + 2 * q], s[half * 64 + 2 * q + 1]), c2, n2);
                    float2 e;
                    if ((q & 7) < FWD_POLY_PAIRS)
                        e = exp2_poly3_x2(x);
                    else
                        e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                    acc[q & 3] = fadd2(acc[q & 3], e);
                    pk[q] = pack_bf16x2(e.x, e.y);
                }
                tmem_st32(tS + half * 32, pk);
            }
            const float2 acc2 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
            const float sum = acc2.x + acc2.y;
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
        // O / l as bf16 goes through this tile's Q buffer, which every MMA that read it has
        // finished with (the tile's last Q K^T precedes its last P V, whose completion O_FINAL
        // signals): each thread writes its row in the tensor map's 128-byte-swizzled layout, then
        // one thread stores the tile with two TMA stores (rows past S are not written).
        const uint32_t stage = sQ + t * TILE_BYTES;
        if (ok) {
            tc_fence_after();
            const float inv_l = 1.f / l;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t o[64];
                tmem_ld32(tO + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
                tmem_ld32(tO + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
                tmem_wait_ld();
                uint32_t w[32];
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
                st_row_sw128(stage + half * HALF_BYTES, r, w);
            }
            fence_proxy_async_smem();
            if (row < p.S)
                p.lse[(static_cast<size_t>(b) * p.H + h) * p.S + row] = (m_ref + log2f(l)) * 0.69314718055994531f;
        }
        named_bar_sync(1 + t, BM);                // every warp of the group, whatever its state
        if (r == 0 && ok && !*abort_flag) {
            tma_store_4d(&tmo, stage, 0, h, q0 + t * BM, b);
            tma_store_4d(&tmo, stage + HALF_BYTES, 64, h, q0 + t * BM, b);
            bulk_commit_group();
            bulk_wait_read_all();                 // the buffer stays valid until the copies have read it
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace fwd

int launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
               const FwdParams& p, cudaStream_t stream) {
    if (configure_smem(reinterpret_cast<const void*>(fwd::attn_fwd_kernel), fwd::SMEM_BYTES) != 0) return -1;
    const dim3 grid((p.S + fwd::NQ * fwd::BM - 1) / (fwd::NQ * fwd::BM), p.H, p.B);
    fwd::attn_fwd_kernel<<<grid, fwd::NTHREADS, fwd::SMEM_BYTES, stream>>>(tq, tk, tv, to, p);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace wan
