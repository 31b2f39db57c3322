// The per-tile bf16 forwards of the Wan DiT attention on sm_100a: the block-sparse forward with
// a given 64 x 64 block mask, O = softmax over each row's allowed keys of Q K^T / sqrt(D),
// times V, and the LSE; and the dense forward over a short key sequence.
//
// The pages: the FastWan / VSA article on the first page: video sparse attention keeps, for
// each 64-token query block, a subset of the 64-token key blocks (87.5 % sparsity in its
// scaling runs) and compares against FlexAttention on the same 64 x 64 block-sparse mask.
// The mask is an input here; the learned coarse stage that picks the blocks is not built.
// The short key sequence is the cross-attention to the text embedding ("Wan 2.1 ...
// paper-podcast summary", section "干预与形式化": cross-attention from the video tokens to the
// umT5 text tokens).
//
// Two kernels, one CTA per 128-row Q tile (2 query blocks of one (b, h)):
//   sparse_tile_lists      one warp per (b, h, Q tile): the ascending union of the key blocks
//                          the tile's 2 query blocks attend, each entry carrying which of
//                          the two attends it, and the union's length.
//   pair::attn_fwd_pair    128-key steps, in a block-sparse form over the lists and a dense
//                          form over every key block (described with the kernel below).
#include <cuda.h>

#include "sm100_ptx.cuh"
#include "wan_attn_internal.h"

namespace wan {
namespace sparse {

constexpr int BM = 128;                       // query rows per CTA (2 query blocks)
constexpr int BK = 64;                        // keys per block
constexpr int HD = 128;
constexpr int Q_BYTES = BM * HD * 2;          // 32 KB: two 64-wide halves of d, 16 KB each
constexpr int Q_HALF = Q_BYTES / 2;
constexpr float RESCALE_THRESHOLD = 8.0f;          // log2 units: keep a stale max while p <= 2^8

// 128-key steps: two 64-key blocks per step, so that Q K^T runs at N = 128.  One kernel, one CTA
// per 128-row Q tile; DENSE = false walks a tile's list, DENSE = true every key block; SMALL
// picks the configuration.  The block-sparse call runs <false, false>, the short-key dense call
// <true, true>.  (The lists on the small configuration measured 26.8 vs 23.5 ms at 720p with
// 1/8 of the blocks.)
//
// Block-sparse configuration (SMALL = false), one CTA per SM.  Step k covers the tile's listed
// key blocks 2k and 2k + 1 (an odd list repeats its last block, which no row then keeps): K and
// V of the pair fill one 128-key stage, S(k) = Q K(k)^T is one N = 128 product into TMEM
// buffer k % 3, and O += P(k) V(k) one K = 128 product.  Three S buffers (with O, all 512 TMEM
// columns) let the chain softmax(k) -> P(k) V(k) -> S(k + 3) span three steps.
//   warps 0-3   softmax, one row per thread: a warp's 32 rows lie in one query block; each
//               half of a step is either attended (keys past Skv masked) or gets P = 0
//               without exponentials.  Online max and sum in fp32 with exp2, the running
//               max moved only when it rises by more than 2^8 (O rescaled in TMEM then);
//               epilogue O / l -> bf16 through the Q buffer and two TMA stores, LSE.
//   warp 4      TMA: Q once, then per step the pair's K (four 8 KB boxes), three stages
//   warp 6      TMA: per step the pair's V, two stages
//   warp 7      tcgen05: S(k) = Q K(k)^T once P(k - 3) V(k - 3) has completed
//   warp 5      tcgen05: O += P(k) V(k) (P bf16 over the first 64 columns of S(k))
// The two MMA threads sit on two sub-partitions: each MMA issue costs its thread more cycles
// than the MMA takes on the tensor core.
//
// Small configuration (SMALL = true), two CTAs per SM, each with half of the tensor memory (one
// S buffer and O) and one stage each of K and V: the same softmax warps, holding one 64-key
// half in registers; warp 4 loads Q, K and V, warp 5 issues S(k), then P(k) V(k), then
// S(k + 1) into the buffer P(k) was read from (tcgen05 MMAs of one thread run in order).  The
// two CTAs on an SM hide each other's softmax, prologue and epilogue.
namespace pair {
constexpr int BN = 128;                                   // keys per step: two key blocks
constexpr int KV_BYTES = BN * HD * 2;                     // 32 KB: [d half][128 keys][128 B]
constexpr int KV_DHALF = KV_BYTES / 2;                    // 16 KB between the two halves of d
constexpr int BLOCK_BYTES = 64 * 128;                     // one key block of one half of d
constexpr unsigned ATTEND0 = 1u << 30, ATTEND1 = 1u << 31, KB_MASK = ATTEND0 - 1u;   // list entries

template <bool SMALL>
struct Cfg {
    static constexpr int NBUF = SMALL ? 1 : 3;            // S buffers in TMEM
    static constexpr int K_STAGES = SMALL ? 1 : 3, V_STAGES = SMALL ? 1 : 2;
    static constexpr int NTHREADS = SMALL ? 192 : 256;
    static constexpr int MIN_CTAS = SMALL ? 2 : 1;        // CTAs per SM
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + K_STAGES * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + V_STAGES * KV_BYTES;
    // barriers: Q; K full / empty per stage; V full / empty per stage; S full, P full and P V
    // done per S buffer; O final; the two MMA threads' drains
    static constexpr int Q_FULL = 0, K_FULL = 1, K_EMPTY = K_FULL + K_STAGES, V_FULL = K_EMPTY + K_STAGES,
                         V_EMPTY = V_FULL + V_STAGES, S_FULL = V_EMPTY + V_STAGES, P_FULL = S_FULL + NBUF,
                         PV_DONE = P_FULL + NBUF, O_FINAL = PV_DONE + NBUF, DRAIN = O_FINAL + 1,
                         DRAIN_QK = DRAIN + 1, NBARS = DRAIN_QK + 1;
    static constexpr int OFF_TMEM_SLOT = OFF_BAR + NBARS * 8;
    static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
    static constexpr int SMEM_BYTES = OFF_ABORT + 8 + 1024;
    static constexpr uint32_t T_O = NBUF * BN;
    static constexpr uint32_t TMEM_COLS = T_O + HD;
    static_assert(K_STAGES <= 3 && V_STAGES <= 3, "the producers track up to three stages per ring");
    static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM is allocated in powers of two");
    static_assert(SMEM_BYTES <= 232448 / MIN_CTAS, "shared memory for MIN_CTAS CTAs per SM");
};
constexpr int WARP_TMA_K = 4, WARP_PV = 5, WARP_TMA_V = 6, WARP_QK = 7;   // sparse roles; dense: 4 TMA, 5 MMA

// Max of 64 scores, those from index lim on taken as -inf (-inf if lim = 0); overwrites them.
__device__ __forceinline__ float masked_max64(float* sc, int lim) {
    if (lim < BK) {
#pragma unroll
        for (int q = 0; q < BK; ++q)
            if (q >= lim) sc[q] = -INFINITY;
    }
    float m4[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) m4[q] = fmax3(sc[q], sc[q + 4], sc[q + 8]);
#pragma unroll
    for (int e = 12; e + 8 <= BK; e += 8)
#pragma unroll
        for (int q = 0; q < 4; ++q) m4[q] = fmax3(m4[q], sc[e + q], sc[e + 4 + q]);
#pragma unroll
    for (int q = 0; q < 4; ++q) m4[q] = fmaxf(m4[q], sc[60 + q]);
    return fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
}

// p = 2^(s c - m) of 64 scores (neg = -m), packed to bf16 pairs; returns their sum.
__device__ __forceinline__ float exp_pack64(const float* sc, float c, float neg, uint32_t (&pk)[32]) {
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < 32; ++q) {
        const float p0 = ex2_approx(fmaf(sc[2 * q], c, neg));
        const float p1 = ex2_approx(fmaf(sc[2 * q + 1], c, neg));
        sum += p0 + p1;
        pk[q] = pack_bf16x2(p0, p1);
    }
    return sum;
}

template <bool DENSE, bool SMALL>
__global__ void __launch_bounds__(Cfg<SMALL>::NTHREADS, Cfg<SMALL>::MIN_CTAS)
attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
                     const FwdParams p) {
    using C = Cfg<SMALL>;
    constexpr int NBUF = C::NBUF, K_STAGES = C::K_STAGES, V_STAGES = C::V_STAGES;
    constexpr int Q_FULL = C::Q_FULL, K_FULL = C::K_FULL, K_EMPTY = C::K_EMPTY, V_FULL = C::V_FULL,
                  V_EMPTY = C::V_EMPTY, S_FULL = C::S_FULL, P_FULL = C::P_FULL, PV_DONE = C::PV_DONE,
                  O_FINAL = C::O_FINAL, DRAIN = C::DRAIN, DRAIN_QK = C::DRAIN_QK;
    constexpr uint32_t T_O = C::T_O, TMEM_COLS = C::TMEM_COLS;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_addr);

    const int warp = warp_id();
    const int lane = lane_id();
    const int h = blockIdx.y, b = blockIdx.z;
    const int q0 = blockIdx.x * BM;
    const size_t li = (static_cast<size_t>(b) * p.H + h) * p.nctas + blockIdx.x;
    const int* list = DENSE ? nullptr : p.kv_list + li * p.nkb;
    const int n = DENSE ? p.nkb : p.kv_count[li];     // key blocks this tile attends
    const int nsteps = (n + 1) / 2;
    // list entry i: the key block with the attend bits of the tile's two query blocks (0 past
    // the list: the repeat of an odd list's last block); every block in the dense form
    auto entry_of = [&](int i) -> unsigned {
        if (i >= n) return 0u;
        return DENSE ? static_cast<unsigned>(i) | ATTEND0 | ATTEND1 : static_cast<unsigned>(list[i]);
    };
    auto block_of = [&](int i) {
        return DENSE ? min(i, n - 1) : static_cast<int>(static_cast<unsigned>(list[min(i, n - 1)]) & KB_MASK);
    };

    const uint32_t sQ = base + C::OFF_Q, sK = base + C::OFF_K, sV = base + C::OFF_V;
    const uint32_t bar0 = base + C::OFF_BAR;
    auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_ABORT);
    const WaitCtl wc{abort_flag, p.wait_budget_ns, p.status};

    if (threadIdx.x == 0) {
        mbar_init(bar(Q_FULL), 1);
        for (int s = 0; s < K_STAGES; ++s) {
            mbar_init(bar(K_FULL + s), 1);
            mbar_init(bar(K_EMPTY + s), 1);
        }
        for (int s = 0; s < V_STAGES; ++s) {
            mbar_init(bar(V_FULL + s), 1);
            mbar_init(bar(V_EMPTY + s), 1);
        }
        for (int s = 0; s < NBUF; ++s) {
            mbar_init(bar(S_FULL + s), 1);
            mbar_init(bar(P_FULL + s), BM);
            mbar_init(bar(PV_DONE + s), 1);
        }
        mbar_init(bar(O_FINAL), 1);
        mbar_init(bar(DRAIN), 1);
        mbar_init(bar(DRAIN_QK), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == WARP_PV) {
        tmem_alloc(base + C::OFF_TMEM_SLOT, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + C::OFF_TMEM_SLOT);
    constexpr uint32_t STAGE16 = KV_BYTES >> 4;

    if (warp == WARP_TMA_K || (!SMALL && warp == WARP_TMA_V)) {
        // ----------------- TMA producers (dense: one thread for Q, K and V) -----------------
        if (lane == 0 && n > 0) {
            const bool do_k = warp == WARP_TMA_K, do_v = SMALL || warp == WARP_TMA_V;
            const uint64_t keep = l2_policy_evict_last();
            if (do_k) {
                tma_prefetch_desc(&tmq);
                tma_prefetch_desc(&tmk);
                mbar_arrive_expect_tx(bar(Q_FULL), Q_BYTES);
                tma_load_4d(sQ, &tmq, bar(Q_FULL), 0, h, q0, b);
                tma_load_4d(sQ + Q_HALF, &tmq, bar(Q_FULL), 64, h, q0, b);
            }
            if (do_v) tma_prefetch_desc(&tmv);
            // a step's two key blocks into one stage: rows 0-63 and 64-127 of each half of d
            auto load_pair = [&](const CUtensorMap* tm, uint32_t dst, uint32_t full, int key_a, int key_b) {
                mbar_arrive_expect_tx(full, KV_BYTES);
                tma_load_4d_hint(dst, tm, full, 0, h, key_a, b, keep);
                tma_load_4d_hint(dst + BLOCK_BYTES, tm, full, 0, h, key_b, b, keep);
                tma_load_4d_hint(dst + KV_DHALF, tm, full, 64, h, key_a, b, keep);
                tma_load_4d_hint(dst + KV_DHALF + BLOCK_BYTES, tm, full, 64, h, key_b, b, keep);
            };
            int kpar[3] = {-1, -1, -1}, vpar[3] = {-1, -1, -1};   // parity of the last copy per stage
            bool ok = true;
            for (int k = 0; k < nsteps && ok; ++k) {
                const int key_a = block_of(2 * k) * BK, key_b = block_of(2 * k + 1) * BK;
                if (do_k) {
                    const int st = k % K_STAGES, use = (k / K_STAGES) & 1;
                    ok = wait_thread(bar(K_EMPTY + st), use ^ 1, wc);
                    if (!ok) break;
                    load_pair(&tmk, sK + st * KV_BYTES, bar(K_FULL + st), key_a, key_b);
                    kpar[st] = use;
                }
                if (do_v) {
                    const int st = k % V_STAGES, use = (k / V_STAGES) & 1;
                    ok = wait_thread(bar(V_EMPTY + st), use ^ 1, wc);
                    if (!ok) break;
                    load_pair(&tmv, sV + st * KV_BYTES, bar(V_FULL + st), key_a, key_b);
                    vpar[st] = use;
                }
            }
            if (!ok) {
                // let the copies already issued land before the CTA's shared memory goes away
                if (do_k) drain_wait(bar(Q_FULL), 0);
                for (int st = 0; st < K_STAGES; ++st)
                    if (kpar[st] >= 0) drain_wait(bar(K_FULL + st), kpar[st]);
                for (int st = 0; st < V_STAGES; ++st)
                    if (vpar[st] >= 0) drain_wait(bar(V_FULL + st), vpar[st]);
            }
        }
    } else if (warp == WARP_PV || (!SMALL && warp == WARP_QK)) {
        // ------------- tcgen05 issuers (dense: one thread for both products) -------------
        if (lane == 0 && n > 0) {
            const bool do_qk = SMALL || warp == WARP_QK, do_pv = SMALL || warp == WARP_PV;
            const uint32_t idesc_qk = make_idesc(1, 1, 1, 0, 0, BM, BN);
            const uint32_t idesc_pv = make_idesc(1, 1, 1, 0, 1, BM, HD);
            const uint32_t hi = sdesc_hi();           // descriptors: common high half, low halves
            const uint32_t q_lo = sdesc_lo(sQ, 16), k_lo = sdesc_lo(sK, 16), v_lo = sdesc_lo(sV, KV_DHALF);
            static_assert(Q_HALF == KV_DHALF, "Q and K tiles share the offset of their second half of d");
            bool ok = true;
            if (do_qk) ok = wait_thread(bar(Q_FULL), 0, wc);
            auto issue_qk = [&](int k) {
                const int sb = k % NBUF, ks = k % K_STAGES;
                // S(k) overwrites the buffer P(k - NBUF) was read from: with one issuing thread the
                // MMAs run in order; with two, wait for that product
                bool good = true;
                if (!SMALL && k >= NBUF) good = wait_thread(bar(PV_DONE + sb), ((k - NBUF) / NBUF) & 1, wc);
                if (good) good = wait_thread(bar(K_FULL + ks), (k / K_STAGES) & 1, wc);
                if (!good) return false;
                tc_fence_after();
                mma8_f16_ss<KV_DHALF / 16, 2>(tmem + static_cast<uint32_t>(sb * BN), q_lo, k_lo + ks * STAGE16, hi,
                                              idesc_qk, 0u);
                mma_commit(bar(S_FULL + sb));
                mma_commit(bar(K_EMPTY + ks));
                return true;
            };
            auto issue_pv = [&](int k) {
                const int sb = k % NBUF, vs = k % V_STAGES;
                bool good = wait_thread(bar(V_FULL + vs), (k / V_STAGES) & 1, wc);
                if (good) good = wait_thread(bar(P_FULL + sb), (k / NBUF) & 1, wc);
                if (!good) return false;
                tc_fence_after();
                // P: 8 columns per 16 keys; V: 2048 bytes per 16 keys, the second block 8 KB on
                mma8_f16_ts<32, BLOCK_BYTES / 16, 128>(tmem + T_O, tmem + static_cast<uint32_t>(sb * BN),
                                                       v_lo + vs * STAGE16, hi, idesc_pv, k > 0 ? 1u : 0u);
                mma_commit(bar(V_EMPTY + vs));
                mma_commit(bar(PV_DONE + sb));
                if (k + 1 == nsteps) mma_commit(bar(O_FINAL));
                return true;
            };
            if (SMALL) {
                if (ok) ok = issue_qk(0);
                for (int k = 0; k < nsteps && ok; ++k) {
                    ok = issue_pv(k);
                    if (ok && k + 1 < nsteps) ok = issue_qk(k + 1);
                }
            } else if (do_qk) {
                for (int k = 0; k < nsteps && ok; ++k) ok = issue_qk(k);
            } else if (do_pv) {
                for (int k = 0; k < nsteps && ok; ++k) ok = issue_pv(k);
            }
            const uint32_t drain = bar(do_pv ? DRAIN : DRAIN_QK);
            mma_commit(drain);
            drain_wait(drain, 0);
        }
    } else {
        // ------------------------- softmax / correction / epilogue ----------------
        const int r = threadIdx.x;                    // row within the tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t tO = tmem + T_O + lane_off;
        const int row = q0 + r;
        const float c = p.scale_log2;
        const unsigned attend = (warp & 2) ? ATTEND1 : ATTEND0;   // the warp's query block's bit
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        // keys of the entry's block this warp's rows keep: 0 if their query block skips it
        auto keep_of = [&](unsigned e) {
            return (e & attend) ? min(BK, p.Skv - BK * static_cast<int>(e & KB_MASK)) : 0;
        };
        unsigned e0 = entry_of(0), e1 = entry_of(1);
        for (int k = 0; k < nsteps && ok; ++k) {
            const unsigned n0 = entry_of(2 * k + 2), n1 = entry_of(2 * k + 3);   // in flight during step k
            const int lim0 = keep_of(e0), lim1 = keep_of(e1);
            const int sb = k % NBUF;
            ok = wait_warp(bar(S_FULL + sb), (k / NBUF) & 1, wc);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tS = tmem + static_cast<uint32_t>(sb * BN) + lane_off;
            float alpha = 1.f, sum = 0.f;
            bool moved = false;
            if constexpr (SMALL) {
                // Registers hold one 64-key half: the max pass loads half 1, then half 0, and the
                // last one loaded stays.  P of half 0 goes over S columns 0-31; half 1 (columns
                // 64-127, untouched) is loaded again if needed and its P goes over columns 32-63,
                // whose scores are then used.
                uint32_t pk[32];
                if (lim0 > 0 || lim1 > 0) {               // warp-uniform
                    uint32_t sr[64];
                    float* sc = reinterpret_cast<float*>(sr);
                    float mx = -INFINITY;
#pragma unroll 1
                    for (int hf = 1; hf >= 0; --hf) {
                        const int lim = hf ? lim1 : lim0;
                        if (lim > 0) {
                            tmem_ld32(tS + hf * 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                            tmem_ld32(tS + hf * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                            tmem_wait_ld();
                            mx = fmaxf(mx, masked_max64(sc, lim));
                        }
                    }
                    const float m_cand = mx * c;      // finite: a half kept
                    if (m_cand > m_ref + RESCALE_THRESHOLD) {
                        alpha = ex2_approx(m_ref - m_cand);
                        m_ref = m_cand;
                        moved = true;
                    }
                    const float neg = -m_ref;
                    if (lim0 > 0) {                   // half 0 in registers
                        sum += exp_pack64(sc, c, neg, pk);
                        tmem_st32(tS, pk);
                        if (lim1 > 0) {
                            tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                            tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                            tmem_wait_ld();
                            masked_max64(sc, lim1);   // masks keys past Skv again
                            sum += exp_pack64(sc, c, neg, pk);
                        } else {
#pragma unroll
                            for (int q = 0; q < 32; ++q) pk[q] = 0u;
                        }
                        tmem_st32(tS + 32, pk);
                    } else {                          // half 1 only, in registers
                        sum += exp_pack64(sc, c, neg, pk);
                        tmem_st32(tS + 32, pk);
#pragma unroll
                        for (int q = 0; q < 32; ++q) pk[q] = 0u;
                        tmem_st32(tS, pk);
                    }
                } else {
                    // P V reads every row of the tile: this one contributes nothing
#pragma unroll
                    for (int q = 0; q < 32; ++q) pk[q] = 0u;
                    tmem_st32(tS, pk);
                    tmem_st32(tS + 32, pk);
                }
            } else if (lim0 > 0 || lim1 > 0) {                   // warp-uniform
                uint32_t sr[128];
                if (lim0 > 0) {
                    tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                    tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                }
                if (lim1 > 0) {
                    tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
                    tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
                }
                tmem_wait_ld();
                float* sc = reinterpret_cast<float*>(sr);
                // an unattended half takes no part in the max; keys past Skv are masked
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int lim = hf ? lim1 : lim0;
                    if (lim < BK) {
#pragma unroll
                        for (int q = 0; q < BK; ++q)
                            if (q >= lim) sc[hf * BK + q] = -INFINITY;
                    }
                }
                float m4[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) m4[q] = fmax3(sc[q], sc[q + 4], sc[q + 8]);
#pragma unroll
                for (int e = 12; e + 8 <= BN; e += 8)
#pragma unroll
                    for (int q = 0; q < 4; ++q) m4[q] = fmax3(m4[q], sc[e + q], sc[e + 4 + q]);
#pragma unroll
                for (int q = 0; q < 4; ++q) m4[q] = fmaxf(m4[q], sc[124 + q]);
                const float m_cand = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3])) * c;   // finite: a half kept
                if (m_cand > m_ref + RESCALE_THRESHOLD) {
                    alpha = ex2_approx(m_ref - m_cand);
                    m_ref = m_cand;
                    moved = true;
                }
                const float neg = -m_ref;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t pk[32];
                    if (hf ? lim1 > 0 : lim0 > 0) {
#pragma unroll
                        for (int q = 0; q < 32; ++q) {
                            const float p0 = ex2_approx(fmaf(sc[hf * BK + 2 * q], c, neg));
                            const float p1 = ex2_approx(fmaf(sc[hf * BK + 2 * q + 1], c, neg));
                            sum += p0 + p1;
                            pk[q] = pack_bf16x2(p0, p1);
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < 32; ++q) pk[q] = 0u;
                    }
                    tmem_st32(tS + hf * 32, pk);          // P (bf16) over S's first 64 columns
                }
            } else {
                // P V reads every row of the tile: this one contributes nothing
                uint32_t pk[32];
#pragma unroll
                for (int q = 0; q < 32; ++q) pk[q] = 0u;
                tmem_st32(tS, pk);
                tmem_st32(tS + 32, pk);
            }
            l = l * alpha + sum;
            if (k > 0 && __any_sync(0xffffffffu, moved)) {
                // O must hold P(k - 1) V(k - 1) before it is rescaled
                const int pb = (k - 1) % NBUF;
                ok = wait_warp(bar(PV_DONE + pb), ((k - 1) / NBUF) & 1, wc);
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
            mbar_arrive(bar(P_FULL + sb));
            e0 = n0;
            e1 = n1;
        }
        if (ok && nsteps > 0) ok = wait_warp(bar(O_FINAL), 0, wc);
        // O / l as bf16 goes through the Q buffer, which every MMA that read it has finished
        // with (the last Q K^T precedes the last P V's P, whose product O_FINAL signals; with
        // no key block nothing was loaded into it): each thread writes its row in the tensor
        // map's 128-byte-swizzled layout, then one thread stores the tile with two TMA stores
        // (rows past S are not written).
        if (ok) {
            tc_fence_after();
            const bool empty = !(l > 0.f);            // no allowed key: O = 0, LSE = -inf
            const float inv_l = empty ? 0.f : 1.f / l;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t w[32];
                if (nsteps > 0 && !empty) {
                    uint32_t o[64];
                    tmem_ld32(tO + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
                    tmem_ld32(tO + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) w[e] = 0u;
                }
                st_row_sw128(sQ + half * Q_HALF, r, w);
            }
            fence_proxy_async_smem();
            if (row < p.S)
                p.lse[(static_cast<size_t>(b) * p.H + h) * p.S + row] =
                    empty ? -INFINITY : (m_ref + log2f(l)) * 0.69314718055994531f;
        }
        named_bar_sync(1, BM);                        // every softmax warp, whatever its state
        if (r == 0 && ok && !*abort_flag) {
            tma_store_4d(&tmo, sQ, 0, h, q0, b);
            tma_store_4d(&tmo, sQ + Q_HALF, 64, h, q0, b);
            bulk_commit_group();
            bulk_wait_read_all();
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == WARP_PV) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace pair

// One warp per (b, h, Q tile): ballot 32 key blocks at a time over the tile's (up to) 2 query
// blocks, writing the ascending union and its length.  Each entry is the key block with bit 30
// set if the tile's first query block attends it and bit 31 if the second does.
__global__ void __launch_bounds__(256) sparse_tile_lists_kernel(const uint8_t* __restrict__ mask,
                                                                int* __restrict__ list, int* __restrict__ count,
                                                                long long nlists, int ntiles, int nqb, int nkb) {
    const int lane = threadIdx.x & 31;
    const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    for (long long w = warp; w < nlists; w += nwarps) {          // w = (b * H + h) * ntiles + tile
        const long long bh = w / ntiles;
        const int tile = static_cast<int>(w - bh * ntiles);
        const int qb0 = tile * 2, nrows = min(2, nqb - qb0);
        const uint8_t* m = mask + (bh * nqb + qb0) * nkb;
        int* out = list + w * nkb;
        int cnt = 0;
        for (int k0 = 0; k0 < nkb; k0 += 32) {
            const int kb = k0 + lane;
            bool r0 = false, r1 = false;
            if (kb < nkb) {
                r0 = m[kb] != 0;
                if (nrows > 1) r1 = m[static_cast<long long>(nkb) + kb] != 0;
            }
            const bool any = r0 || r1;
            const unsigned bal = __ballot_sync(0xffffffffu, any);
            if (any)
                out[cnt + __popc(bal & ((1u << lane) - 1u))] =
                    static_cast<int>(static_cast<unsigned>(kb) | (r0 ? pair::ATTEND0 : 0u) | (r1 ? pair::ATTEND1 : 0u));
            cnt += __popc(bal);
        }
        if (lane == 0) count[w] = cnt;
    }
}

}  // namespace sparse

int launch_fwd_tiles(const CUtensorMap& tq, const CUtensorMap& tk64, const CUtensorMap& tv64, const CUtensorMap& to,
                     const FwdParams& p, cudaStream_t stream) {
    if (p.kv_list) {
        int sms = 148, dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const long long nlists = static_cast<long long>(p.B) * p.H * p.nctas;
        sparse::sparse_tile_lists_kernel<<<sms * 8, 256, 0, stream>>>(p.mask, const_cast<int*>(p.kv_list),
                                                                      const_cast<int*>(p.kv_count), nlists, p.nctas,
                                                                      p.nqb, p.nkb);
        if (cudaGetLastError() != cudaSuccess) return -1;
    }
    const dim3 grid(p.nctas, p.H, p.B);
    auto run = [&](auto kernel, int threads, int smem) {
        if (configure_smem(reinterpret_cast<const void*>(kernel), smem) != 0) return -1;
        kernel<<<grid, threads, smem, stream>>>(tq, tk64, tv64, to, p);
        return cudaGetLastError() == cudaSuccess ? 0 : -1;
    };
    using sparse::pair::Cfg;
    if (p.kv_list)
        return run(sparse::pair::attn_fwd_pair_kernel<false, false>, Cfg<false>::NTHREADS, Cfg<false>::SMEM_BYTES);
    return run(sparse::pair::attn_fwd_pair_kernel<true, true>, Cfg<true>::NTHREADS, Cfg<true>::SMEM_BYTES);
}

}  // namespace wan
