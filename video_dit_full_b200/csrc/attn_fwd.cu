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
//               written back to TMEM as bf16; epilogue O / l -> bf16, LSE.
// The two Q tiles ping-pong: while one softmax group works on its S, the
// tensor core runs the other tile's P V and Q K^T.
//
// Block-sparse form (template SPARSE): a 64 x 64 block mask selects, for each
// 64-token query block, the 64-token key blocks it attends (the FastWan / VSA
// article on the first page: 64 x 64 block-sparse masks).  A CTA walks only
// the key blocks that any of its 4 query blocks attends, two blocks per K/V
// stage (each TMA-loaded into one 64-row half, wherever it lies); the softmax
// sets each row's disallowed halves to -inf.  A row that attends nothing gets
// O = 0 and LSE = -inf.
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
// Sparse list entries: the key block in the low bits, and whether Q tile 0 / 1 of the CTA (its
// query blocks 0-1 / 2-3) attends it in bits 28 / 29.
constexpr int KB_BITS = (1 << 28) - 1;
constexpr int NEED_SHIFT = 28;
constexpr float RESCALE_THRESHOLD = 8.0f;      // log2 units: keep a stale max while p <= 2^8

__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_smem, uint32_t k_smem, uint32_t idesc) {
    // K = 128 = 8 steps of 16; steps 0-3 in the first 64-column half, 4-7 in the second.
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
        const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
        mma_f16_ss(d_tmem, sdesc_sw128(q_smem + off, 16, 1024), sdesc_sw128(k_smem + off, 16, 1024), idesc,
                   kk > 0 ? 1u : 0u);
    }
}

// O += P V over the 16-key steps [kk0, kk1) of the tile (0-4: the first 64 keys, 4-8: the
// second).  A = P (128 x 128 bf16 in TMEM, 2 per column), B = V stored [key][d] (MN-major):
// 16 keys per step = 2048 bytes; the two 64-wide halves of d are 16 KB apart (LBO).  The first
// MMA accumulates onto O only if `accumulate`.
__device__ __forceinline__ void issue_pv_keys(uint32_t d_tmem, uint32_t p_tmem, uint32_t v_smem, uint32_t idesc,
                                              bool accumulate, int kk0, int kk1) {
    for (int kk = kk0; kk < kk1; ++kk) {
        mma_f16_ts(d_tmem, p_tmem + kk * 8, sdesc_sw128(v_smem + kk * 2048, HALF_BYTES, 1024), idesc,
                   (accumulate || kk > kk0) ? 1u : 0u);
    }
}

template <bool SPARSE>
__global__ void __launch_bounds__(NTHREADS, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                const __grid_constant__ CUtensorMap tmv, const FwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_addr);

    const int warp = warp_id();
    const int lane = lane_id();
    const int h = blockIdx.y, b = blockIdx.z;
    const int q0 = blockIdx.x * (NQ * BM);
    const int nq = (q0 + BM < p.S) ? 2 : 1;          // second tile empty on a short tail
    // sparse: this CTA's key blocks, two per K/V step
    const int* kv_list = nullptr;
    int kv_count = 0;
    if constexpr (SPARSE) {
        const size_t li = (static_cast<size_t>(b) * p.H + h) * p.nctas + blockIdx.x;
        kv_list = p.kv_list + li * p.nkb;
        kv_count = p.kv_count[li];
    }
    const int nkv = SPARSE ? (kv_count + 1) / 2 : (p.Skv + BN - 1) / BN;

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
        if (lane == 0 && nkv > 0) {
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
                if constexpr (SPARSE) {
                    // two 64-key blocks into rows 0-63 and 64-127 of both 64-wide halves of d (a missing
                    // second block repeats the first; the softmax masks it)
                    const int ka = (kv_list[2 * j] & KB_BITS) * 64;
                    const int kb = (kv_list[min(2 * j + 1, kv_count - 1)] & KB_BITS) * 64;
                    for (int e = 0; e < 2; ++e) {
                        const uint32_t dst = sK + s * TILE_BYTES + e * HALF_BYTES;
                        tma_load_4d_hint(dst, &tmk, bar(K_FULL + s), 64 * e, h, ka, b, keep);
                        tma_load_4d_hint(dst + HALF_BYTES / 2, &tmk, bar(K_FULL + s), 64 * e, h, kb, b, keep);
                    }
                } else {
                    tma_load_4d_hint(sK + s * TILE_BYTES, &tmk, bar(K_FULL + s), 0, h, j * BN, b, keep);
                    tma_load_4d_hint(sK + s * TILE_BYTES + HALF_BYTES, &tmk, bar(K_FULL + s), 64, h, j * BN, b, keep);
                }
                kpar[s] = use;
                ok = wait_thread(bar(V_EMPTY + s), use ^ 1, wc);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(V_FULL + s), TILE_BYTES);
                if constexpr (SPARSE) {
                    const int ka = (kv_list[2 * j] & KB_BITS) * 64;
                    const int kb = (kv_list[min(2 * j + 1, kv_count - 1)] & KB_BITS) * 64;
                    for (int e = 0; e < 2; ++e) {
                        const uint32_t dst = sV + s * TILE_BYTES + e * HALF_BYTES;
                        tma_load_4d_hint(dst, &tmv, bar(V_FULL + s), 64 * e, h, ka, b, keep);
                        tma_load_4d_hint(dst + HALF_BYTES / 2, &tmv, bar(V_FULL + s), 64 * e, h, kb, b, keep);
                    }
                } else {
                    tma_load_4d_hint(sV + s * TILE_BYTES, &tmv, bar(V_FULL + s), 0, h, j * BN, b, keep);
                    tma_load_4d_hint(sV + s * TILE_BYTES + HALF_BYTES, &tmv, bar(V_FULL + s), 64, h, j * BN, b, keep);
                }
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
            const uint32_t idesc_qk64 = make_idesc(1, 1, 1, 0, 0, BM, BN / 2);
            const uint32_t idesc_pv = make_idesc(1, 1, 1, 0, 1, BM, HD);
            // Which 64-key halves of step j tile t needs: bit 0 the first block, bit 1 the second.
            // Dense: both.  Sparse: a half none of the tile's query blocks attends is neither
            // computed (Q K^T of the other half alone, N = 64) nor multiplied into O; its S is
            // never read, since every row of the tile has it masked.  The barriers still pass
            // every step, so phases stay in step with the softmax.
            auto need = [&](int j, int t) -> uint32_t {
                if constexpr (!SPARSE) return 3u;
                const uint32_t ea = static_cast<uint32_t>(kv_list[2 * j]);
                const uint32_t eb = 2 * j + 1 < kv_count ? static_cast<uint32_t>(kv_list[2 * j + 1]) : 0u;
                return ((ea >> (NEED_SHIFT + t)) & 1u) | (((eb >> (NEED_SHIFT + t)) & 1u) << 1);
            };
            auto qk = [&](int t, uint32_t k_stage, uint32_t nd) {
                const uint32_t d = tmem + t * BN, qs = sQ + t * TILE_BYTES;
                if (nd == 3u) issue_qk(d, qs, k_stage, idesc_qk);
                else if (nd == 1u) issue_qk(d, qs, k_stage, idesc_qk64);
                else if (nd == 2u) issue_qk(d + BN / 2, qs, k_stage + HALF_BYTES / 2, idesc_qk64);
            };
            bool o_init[2] = {false, false};               // has a P V product written O yet
            auto pv = [&](int t, uint32_t v_stage, uint32_t nd) {
                if (nd == 0u) return;
                issue_pv_keys(tmem + 256 + t * HD, tmem + t * BN, v_stage, idesc_pv, o_init[t],
                              nd & 1u ? 0 : 4, nd & 2u ? 8 : 4);
                o_init[t] = true;
            };
            bool ok = nkv > 0;                           // sparse: a CTA may attend no key block
            for (int t = 0; t < nq && ok; ++t) ok = wait_thread(bar(Q_FULL + t), 0, wc);
            if (ok) ok = wait_thread(bar(K_FULL + 0), 0, wc);
            if (ok) {
                tc_fence_after();
                for (int t = 0; t < nq; ++t) {
                    qk(t, sK, need(0, t));
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
                    pv(t, sV + s * TILE_BYTES, need(j, t));
                    if (j + 1 == nkv) mma_commit(bar(O_FINAL + t));
                    if (j + 1 < nkv) {
                        if (t == 0) {
                            ok = wait_thread(bar(K_FULL + s1), ((j + 1) >> 1) & 1, wc);
                            if (!ok) break;
                            tc_fence_after();
                        }
                        qk(t, sK + s1 * TILE_BYTES, need(j + 1, t));
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
            // keys kept in each 64-column half; in the sparse kernel a half its row does not attend
            // (lim 0) is left out of the max and the exponentials and gets P = 0
            int lim0 = 64, lim1 = 64;
            if constexpr (SPARSE) {
                // the two key blocks of this step: each half keeps its keys if the row's query block
                // attends the block (and the keys exist); a missing second block is masked.  A
                // warp's 32 rows lie in one 64-row query block, so lim0 and lim1 are warp-uniform.
                const int kba = kv_list[2 * j] & KB_BITS;
                const int kbb = (2 * j + 1 < kv_count) ? (kv_list[2 * j + 1] & KB_BITS) : -1;
                const int qb = min(row, p.S - 1) / 64;
                const uint8_t* mrow = p.mask + ((static_cast<size_t>(b) * p.H + h) * p.nqb + qb) * p.nkb;
                lim0 = mrow[kba] ? min(64, p.Skv - 64 * kba) : 0;
                lim1 = (kbb >= 0 && mrow[kbb]) ? min(64, p.Skv - 64 * kbb) : 0;
                if (lim0 > 0 && lim0 < 64) {                       // a short last key block
#pragma unroll
                    for (int q = 0; q < 64; ++q)
                        if (q >= lim0) s[q] = -INFINITY;
                }
                if (lim1 > 0 && lim1 < 64) {
#pragma unroll
                    for (int q = 0; q < 64; ++q)
                        if (q >= lim1) s[64 + q] = -INFINITY;
                }
            } else {
                const int valid = p.Skv - j * BN;    // keys of this tile that exist
                if (valid < BN) {
#pragma unroll
                    for (int q = 0; q < 128; ++q)
                        if (q >= valid) s[q] = -INFINITY;
                }
            }
            // row max of each half: 4 chains of three-input maxima
            auto half_max = [&](int h0) {
                float m4[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) m4[q] = fmax3(s[h0 + q], s[h0 + q + 4], s[h0 + q + 8]);
#pragma unroll
                for (int e = 12; e + 8 <= 64; e += 8)
#pragma unroll
                    for (int q = 0; q < 4; ++q) m4[q] = fmax3(m4[q], s[h0 + e + q], s[h0 + e + 4 + q]);
#pragma unroll
                for (int q = 0; q < 4; ++q) m4[q] = fmaxf(m4[q], s[h0 + 60 + q]);
                return fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
            };
            float mx = -INFINITY;
            if (lim0 > 0) mx = half_max(0);
            if (lim1 > 0) mx = fmaxf(mx, half_max(64));
            const float m_cand = mx * c;
            float alpha = 1.f;
            bool moved = false;
            if (m_cand > m_ref + RESCALE_THRESHOLD) {
                alpha = ex2_approx(m_ref - m_cand);
                m_ref = m_cand;
                moved = true;
            }
            // sparse: until a row meets its first allowed key, m_ref is -inf and every s is -inf;
            // subtracting 0 then keeps exp2(-inf) = 0 instead of exp2(-inf + inf)
            const float neg = (SPARSE && m_ref == -INFINITY) ? 0.f : -m_ref;
            float sum = 0.f;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t pk[32];
                if (SPARSE && (half == 0 ? lim0 : lim1) == 0) {
#pragma unroll
                    for (int q = 0; q < 32; ++q) pk[q] = 0u;
                    tmem_st32(tS + half * 32, pk);
                    continue;
                }
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    const float p0 = ex2_approx(fmaf(s[half * 64 + 2 * q], c, neg));
                    const float p1 = ex2_approx(fmaf(s[half * 64 + 2 * q + 1], c, neg));
                    sum += p0 + p1;
                    pk[q] = pack_bf16x2(p0, p1);
                }
                tmem_st32(tS + half * 32, pk);
            }
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
        if (ok && nkv > 0) ok = wait_warp(bar(O_FINAL + t), 0, wc);
        if (ok) {
            tc_fence_after();
            // sparse: a row with no allowed key (l = 0, or no key block at all) gets O = 0, LSE = -inf
            const bool empty = SPARSE && !(l > 0.f);
            const float inv_l = empty ? 0.f : 1.f / l;
            __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) +
                                  ((static_cast<size_t>(b) * p.S + row) * p.H + h) * HD;
#pragma unroll 1
            for (int q = 0; q < 4; ++q) {
                uint32_t o[32];
                tmem_ld32(tO + q * 32, o);
                tmem_wait_ld();
                uint4 pk[4];
                uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pw[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
                if (empty) {                                   // TMEM O may never have been written
#pragma unroll
                    for (int e = 0; e < 16; ++e) pw[e] = 0u;
                }
                if (row < p.S) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[e] = pk[e];
                }
            }
            if (row < p.S)
                p.lse[(static_cast<size_t>(b) * p.H + h) * p.S + row] =
                    empty ? -INFINITY : (m_ref + log2f(l)) * 0.69314718055994531f;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace fwd

int launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
               cudaStream_t stream) {
    if (configure_smem(reinterpret_cast<const void*>(fwd::attn_fwd_kernel<false>), fwd::SMEM_BYTES) != 0) return -1;
    const dim3 grid((p.S + fwd::NQ * fwd::BM - 1) / (fwd::NQ * fwd::BM), p.H, p.B);
    fwd::attn_fwd_kernel<false><<<grid, fwd::NTHREADS, fwd::SMEM_BYTES, stream>>>(tq, tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

namespace fwd {
// One warp per (b, h, CTA): the ascending key blocks that any of the CTA's 4 query blocks attends
// (a ballot over 32 key blocks at a time).
__global__ void __launch_bounds__(256) sparse_lists_kernel(const uint8_t* __restrict__ mask, int* __restrict__ list,
                                                           int* __restrict__ count, long long nlists, int nctas,
                                                           int nqb, int nkb) {
    const int lane = threadIdx.x & 31;
    const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    for (long long w = warp; w < nlists; w += nwarps) {          // w = (b * H + h) * nctas + cta
        const long long bh = w / nctas;
        const int cta = static_cast<int>(w - bh * nctas);
        const int qb0 = cta * 4, nrows = min(4, nqb - qb0);
        const uint8_t* m = mask + (bh * nqb + qb0) * nkb;
        int* out = list + w * nkb;
        int n = 0;
        for (int k0 = 0; k0 < nkb; k0 += 32) {
            const int kb = k0 + lane;
            int tiles = 0;                                // bit t: Q tile t (query blocks 2t, 2t+1)
            if (kb < nkb)
                for (int r = 0; r < nrows; ++r)
                    if (m[static_cast<long long>(r) * nkb + kb] != 0) tiles |= 1 << (r >> 1);
            const bool any = tiles != 0;
            const unsigned bal = __ballot_sync(0xffffffffu, any);
            if (any) out[n + __popc(bal & ((1u << lane) - 1u))] = kb | (tiles << NEED_SHIFT);
            n += __popc(bal);
        }
        if (lane == 0) count[w] = n;
    }
}
}  // namespace fwd

int launch_fwd_block_sparse(const CUtensorMap& tq, const CUtensorMap& tk64, const CUtensorMap& tv64,
                            const FwdParams& p, cudaStream_t stream) {
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long nlists = static_cast<long long>(p.B) * p.H * p.nctas;
    fwd::sparse_lists_kernel<<<sms * 8, 256, 0, stream>>>(p.mask, const_cast<int*>(p.kv_list),
                                                          const_cast<int*>(p.kv_count), nlists, p.nctas, p.nqb, p.nkb);
    if (cudaGetLastError() != cudaSuccess) return -1;
    if (configure_smem(reinterpret_cast<const void*>(fwd::attn_fwd_kernel<true>), fwd::SMEM_BYTES) != 0) return -1;
    const dim3 grid(p.nctas, p.H, p.B);
    fwd::attn_fwd_kernel<true><<<grid, fwd::NTHREADS, fwd::SMEM_BYTES, stream>>>(tq, tk64, tv64, p);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace wan
