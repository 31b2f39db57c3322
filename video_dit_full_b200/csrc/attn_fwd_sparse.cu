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
// Three kernels, one CTA per 128-row Q tile (2 query blocks of one (b, h)):
//   sparse_tile_lists            one warp per (b, h, Q tile): the ascending union of the key
//                                blocks the tile's 2 query blocks attend, each entry carrying
//                                which of the two attends it, and the union's length.
//   pair::attn_fwd_sparse_pair   the block-sparse forward: two listed key blocks per step
//                                (described with the kernel below).
//   attn_fwd_sparse_kernel       the dense short-key forward: every key block in 64-key steps,
//                                two CTAs per SM, each with half of the tensor memory, so that
//                                at a few key blocks per tile the two hide each other's
//                                prologue and epilogue:
//     warp 4     TMA: the Q tile once, then the 64-key blocks, K and V each into a two-stage
//                ring of 16 KB tiles (128-byte swizzle).
//     warp 5     tcgen05 issuer: S(k) = Q K(k)^T into TMEM buffer k % 2 (N = 64), then
//                O += P(k) V(k) with P read from TMEM (bf16 over S(k)); S(k + 2) is issued
//                right after P(k) V(k), into the buffer P(k) was just read from, so the
//                softmax finds S(k + 1) ready when it finishes step k.
//     warps 0-3  softmax, one row per thread (keys past Skv masked); online max and sum in
//                fp32 with exp2, the running max moved only when it rises by more than 2^8
//                (O rescaled in TMEM then); epilogue O / l -> bf16 through the Q buffer and
//                two TMA stores, LSE.
#include <cuda.h>

#include "sm100_ptx.cuh"
#include "wan_attn_internal.h"

namespace wan {
namespace sparse {

constexpr int BM = 128;                       // query rows per CTA (2 query blocks)
constexpr int BK = 64;                        // keys per step: one key block
constexpr int HD = 128;
constexpr int Q_BYTES = BM * HD * 2;          // 32 KB: two 64-wide halves of d, 16 KB each
constexpr int Q_HALF = Q_BYTES / 2;
constexpr int KV_BYTES = BK * HD * 2;         // 16 KB: two 64-wide halves of d, 8 KB each
constexpr int KV_HALF = KV_BYTES / 2;
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + Q_BYTES;
constexpr int OFF_V = OFF_K + 2 * KV_BYTES;
constexpr int OFF_BAR = OFF_V + 2 * KV_BYTES;
// S_FULL + b / P_FULL + b: S / P of buffer b.  Per-buffer barriers keep every waiter at most
// one phase behind: the softmax may finish steps k and k + 1 before the MMA takes P(k), but
// not step k + 2, whose S is computed only after that.  PV_LAST: P V of the next-to-last
// step has landed in O; O_FINAL: the last one has.
enum Bar { Q_FULL = 0, K_FULL = 1, K_EMPTY = 3, V_FULL = 5, V_EMPTY = 7, S_FULL = 9, P_FULL = 11,
           PV_LAST = 13, O_FINAL = 14, DRAIN = 15, NBARS = 16 };
constexpr int OFF_TMEM_SLOT = OFF_BAR + NBARS * 8;
constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
constexpr int SMEM_BYTES = OFF_ABORT + 8 + 1024;   // slack for the 1024-byte alignment of the tiles
constexpr int NTHREADS = 192;                      // warps 0-3 softmax, 4 TMA, 5 MMA
constexpr uint32_t TMEM_COLS = 256;                // S buffers at 0 and 64, O at 128
constexpr uint32_t T_O = 128;
constexpr float RESCALE_THRESHOLD = 8.0f;          // log2 units: keep a stale max while p <= 2^8

// S (fp32, N = 64) = Q K^T: Q [128 rows][d] and K [64 rows][d], each as two 64-wide halves of
// d with the 128-byte swizzle; K = 16 per MMA, steps 0-3 in the first half, 4-7 in the second.
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_smem, uint32_t k_smem, uint32_t idesc) {
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk)
        mma_f16_ss(d_tmem, sdesc_sw128(q_smem + (kk >> 2) * Q_HALF + (kk & 3) * 32, 16, 1024),
                   sdesc_sw128(k_smem + (kk >> 2) * KV_HALF + (kk & 3) * 32, 16, 1024), idesc, kk > 0 ? 1u : 0u);
}

// O += P V: A = P (128 x 64 bf16 in TMEM, 2 per column), B = V stored [key][d] (MN-major):
// 16 keys per MMA = 2048 bytes; the two 64-wide halves of d are 8 KB apart (LBO).
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint32_t v_smem, uint32_t idesc,
                                         bool accumulate) {
#pragma unroll
    for (int kk = 0; kk < BK / 16; ++kk)
        mma_f16_ts(d_tmem, p_tmem + kk * 8, sdesc_sw128(v_smem + kk * 2048, KV_HALF, 1024), idesc,
                   (accumulate || kk > 0) ? 1u : 0u);
}

__global__ void __launch_bounds__(NTHREADS, 2)
attn_fwd_sparse_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
                       const FwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_addr);

    const int warp = warp_id();
    const int lane = lane_id();
    const int h = blockIdx.y, b = blockIdx.z;
    const int q0 = blockIdx.x * BM;
    const int n = p.nkb;                              // every key block, no mask

    const uint32_t sQ = base + OFF_Q, sK = base + OFF_K, sV = base + OFF_V;
    const uint32_t bar0 = base + OFF_BAR;
    auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
    const WaitCtl wc{abort_flag, p.wait_budget_ns, p.status};

    if (threadIdx.x == 0) {
        mbar_init(bar(Q_FULL), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(K_FULL + s), 1);
            mbar_init(bar(K_EMPTY + s), 1);
            mbar_init(bar(V_FULL + s), 1);
            mbar_init(bar(V_EMPTY + s), 1);
            mbar_init(bar(S_FULL + s), 1);
            mbar_init(bar(P_FULL + s), BM);
        }
        mbar_init(bar(PV_LAST), 1);
        mbar_init(bar(O_FINAL), 1);
        mbar_init(bar(DRAIN), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 5) {
        tmem_alloc(base + OFF_TMEM_SLOT, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEM_SLOT);

    if (warp == 4) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0 && n > 0) {
            tma_prefetch_desc(&tmq);
            tma_prefetch_desc(&tmk);
            tma_prefetch_desc(&tmv);
            const uint64_t keep = l2_policy_evict_last();
            mbar_arrive_expect_tx(bar(Q_FULL), Q_BYTES);
            tma_load_4d(sQ, &tmq, bar(Q_FULL), 0, h, q0, b);
            tma_load_4d(sQ + Q_HALF, &tmq, bar(Q_FULL), 64, h, q0, b);
            int kpar[2] = {-1, -1}, vpar[2] = {-1, -1};   // parity of the last copy issued per stage
            bool ok = true;
            for (int k = 0; k < n && ok; ++k) {
                const int s = k & 1, use = (k >> 1) & 1;
                const int key0 = k * BK;
                ok = wait_thread(bar(K_EMPTY + s), use ^ 1, wc);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(K_FULL + s), KV_BYTES);
                tma_load_4d_hint(sK + s * KV_BYTES, &tmk, bar(K_FULL + s), 0, h, key0, b, keep);
                tma_load_4d_hint(sK + s * KV_BYTES + KV_HALF, &tmk, bar(K_FULL + s), 64, h, key0, b, keep);
                kpar[s] = use;
                ok = wait_thread(bar(V_EMPTY + s), use ^ 1, wc);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(V_FULL + s), KV_BYTES);
                tma_load_4d_hint(sV + s * KV_BYTES, &tmv, bar(V_FULL + s), 0, h, key0, b, keep);
                tma_load_4d_hint(sV + s * KV_BYTES + KV_HALF, &tmv, bar(V_FULL + s), 64, h, key0, b, keep);
                vpar[s] = use;
            }
            if (!ok) {
                // let the copies already issued land before the CTA's shared memory goes away
                drain_wait(bar(Q_FULL), 0);
                for (int s = 0; s < 2; ++s) {
                    if (kpar[s] >= 0) drain_wait(bar(K_FULL + s), kpar[s]);
                    if (vpar[s] >= 0) drain_wait(bar(V_FULL + s), vpar[s]);
                }
            }
        }
    } else if (warp == 5) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0 && n > 0) {
            const uint32_t idesc_qk = make_idesc(1, 1, 1, 0, 0, BM, BK);
            const uint32_t idesc_pv = make_idesc(1, 1, 1, 0, 1, BM, HD);
            auto sbuf = [&](int k) { return tmem + static_cast<uint32_t>((k & 1) * BK); };
            bool ok = wait_thread(bar(Q_FULL), 0, wc);
            for (int k = 0; k < 2 && k < n && ok; ++k) {
                ok = wait_thread(bar(K_FULL + k), 0, wc);
                if (!ok) break;
                tc_fence_after();
                issue_qk(sbuf(k), sQ, sK + k * KV_BYTES, idesc_qk);
                mma_commit(bar(S_FULL + k));
                mma_commit(bar(K_EMPTY + k));
            }
            for (int k = 0; k < n && ok; ++k) {
                const int s = k & 1;
                const bool next = k + 2 < n;              // K(k + 2) goes to stage s too
                ok = wait_thread(bar(V_FULL + s), (k >> 1) & 1, wc);
                if (ok && next) ok = wait_thread(bar(K_FULL + s), ((k + 2) >> 1) & 1, wc);
                if (ok) ok = wait_thread(bar(P_FULL + s), (k >> 1) & 1, wc);
                if (!ok) break;
                tc_fence_after();
                issue_pv(tmem + T_O, sbuf(k), sV + s * KV_BYTES, idesc_pv, k > 0);
                mma_commit(bar(V_EMPTY + s));
                if (k + 2 == n) mma_commit(bar(PV_LAST));
                if (k + 1 == n) mma_commit(bar(O_FINAL));
                if (next) {
                    issue_qk(sbuf(k), sQ, sK + s * KV_BYTES, idesc_qk);
                    mma_commit(bar(S_FULL + s));
                    mma_commit(bar(K_EMPTY + s));
                }
            }
            // every MMA issued so far completes before TMEM is released
            mma_commit(bar(DRAIN));
            drain_wait(bar(DRAIN), 0);
        }
    } else {
        // ------------------------- softmax / correction / epilogue ----------------
        const int r = threadIdx.x;                    // row within the tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t tO = tmem + T_O + lane_off;
        const int row = q0 + r;
        const float c = p.scale_log2;
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        // keys of step k (short for the last key block)
        auto keep_of = [&](int k) { return min(BK, p.Skv - BK * k); };
        int lim_next = n > 0 ? keep_of(0) : 0;
        for (int k = 0; k < n && ok; ++k) {
            const int lim = lim_next;
            ok = wait_warp(bar(S_FULL + (k & 1)), (k >> 1) & 1, wc);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tS = tmem + static_cast<uint32_t>((k & 1) * BK) + lane_off;
            uint32_t pk[32];
            float alpha = 1.f, sum = 0.f;
            bool moved = false;
            uint32_t sr[64];
            tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
            tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
            tmem_wait_ld();
            float* s = reinterpret_cast<float*>(sr);
            if (lim < BK) {
#pragma unroll
                for (int q = 0; q < BK; ++q)
                    if (q >= lim) s[q] = -INFINITY;
            }
            float m4[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) m4[q] = fmax3(s[q], s[q + 4], s[q + 8]);
#pragma unroll
            for (int e = 12; e + 8 <= BK; e += 8)
#pragma unroll
                for (int q = 0; q < 4; ++q) m4[q] = fmax3(m4[q], s[e + q], s[e + 4 + q]);
#pragma unroll
            for (int q = 0; q < 4; ++q) m4[q] = fmaxf(m4[q], s[60 + q]);
            const float m_cand = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3])) * c;   // finite: lim > 0
            if (m_cand > m_ref + RESCALE_THRESHOLD) {
                alpha = ex2_approx(m_ref - m_cand);
                m_ref = m_cand;
                moved = true;
            }
            const float neg = -m_ref;
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const float p0 = ex2_approx(fmaf(s[2 * q], c, neg));
                const float p1 = ex2_approx(fmaf(s[2 * q + 1], c, neg));
                sum += p0 + p1;
                pk[q] = pack_bf16x2(p0, p1);
            }
            tmem_st32(tS, pk);                            // P (bf16) over S's first 32 columns
            l = l * alpha + sum;
            if (k > 0 && __any_sync(0xffffffffu, moved)) {
                // O must hold P(k - 1) V(k - 1) before it is rescaled.  S(k + 1) is computed after
                // that product (one thread issues the MMAs, in order), so its barrier says so;
                // the last step, which has no S(k + 1), has PV_LAST.
                ok = (k + 1 < n) ? wait_warp(bar(S_FULL + ((k + 1) & 1)), ((k + 1) >> 1) & 1, wc)
                                 : wait_warp(bar(PV_LAST), 0, wc);
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
            mbar_arrive(bar(P_FULL + (k & 1)));
            if (k + 1 < n) lim_next = keep_of(k + 1);
        }
        if (ok && n > 0) ok = wait_warp(bar(O_FINAL), 0, wc);
        // O / l as bf16 goes through the Q buffer, which every MMA that read it has finished
        // with (the last Q K^T precedes the last P V, whose completion O_FINAL signals; with no
        // key block nothing was loaded into it): each thread writes its row in the tensor map's
        // 128-byte-swizzled layout, then one thread stores the tile with two TMA stores (rows
        // past S are not written).
        if (ok) {
            tc_fence_after();
            // a row with no allowed key (l = 0, or no key block at all) gets O = 0, LSE = -inf
            const bool empty = !(l > 0.f);
            const float inv_l = empty ? 0.f : 1.f / l;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t w[32];
                if (n > 0) {                               // TMEM O is written only if a step ran
                    uint32_t o[64];
                    tmem_ld32(tO + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
                    tmem_ld32(tO + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
                }
                if (empty) {
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
            bulk_wait_read_all();                     // the buffer stays valid until the copies have read it
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, TMEM_COLS);
}

// The block-sparse path: pairs of listed key blocks per step, so that Q K^T runs at N = 128.
//
// One CTA per SM and per 128-row Q tile.  Step k covers the tile's listed key blocks 2k and
// 2k + 1 (an odd list repeats its last block, which no row then keeps): K and V of the pair
// fill one 128-key stage, S(k) = Q K(k)^T is one N = 128 product into TMEM buffer k % 3, and
// O += P(k) V(k) one K = 128 product.  Three S buffers (with O, all 512 TMEM columns) let the
// chain softmax(k) -> P(k) V(k) -> S(k + 3) span three steps.
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
namespace pair {
constexpr int BN = 128;                                   // keys per step: two key blocks
constexpr int NBUF = 3;                                   // S buffers in TMEM
constexpr int KV_BYTES = BN * HD * 2;                     // 32 KB: [d half][128 keys][128 B]
constexpr int KV_DHALF = KV_BYTES / 2;                    // 16 KB between the two halves of d
constexpr int BLOCK_BYTES = 64 * 128;                     // one key block of one half of d
constexpr int K_STAGES = 3, V_STAGES = 2;
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + Q_BYTES;
constexpr int OFF_V = OFF_K + K_STAGES * KV_BYTES;
constexpr int OFF_BAR = OFF_V + V_STAGES * KV_BYTES;
enum Bar { Q_FULL = 0, K_FULL = 1, K_EMPTY = 4, V_FULL = 7, V_EMPTY = 9, S_FULL = 11, P_FULL = 14,
           PV_DONE = 17, O_FINAL = 20, DRAIN = 21, DRAIN_QK = 22, NBARS = 23 };
constexpr int OFF_TMEM_SLOT = OFF_BAR + NBARS * 8;
constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
constexpr int SMEM_BYTES = OFF_ABORT + 8 + 1024;
constexpr unsigned ATTEND0 = 1u << 30, ATTEND1 = 1u << 31, KB_MASK = ATTEND0 - 1u;   // list entries
constexpr int NTHREADS = 256;
constexpr int WARP_TMA_K = 4, WARP_PV = 5, WARP_TMA_V = 6, WARP_QK = 7;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t T_O = NBUF * BN;

__global__ void __launch_bounds__(pair::NTHREADS, 1)
attn_fwd_sparse_pair_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                            const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
                            const FwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_addr);

    const int warp = warp_id();
    const int lane = lane_id();
    const int h = blockIdx.y, b = blockIdx.z;
    const int q0 = blockIdx.x * BM;
    const size_t li = (static_cast<size_t>(b) * p.H + h) * p.nctas + blockIdx.x;
    const int* list = p.kv_list + li * p.nkb;
    const int n = p.kv_count[li];                     // key blocks this tile attends
    const int nsteps = (n + 1) / 2;
    auto block_of = [&](int i) { return static_cast<int>(static_cast<unsigned>(list[min(i, n - 1)]) & KB_MASK); };

    const uint32_t sQ = base + OFF_Q, sK = base + OFF_K, sV = base + OFF_V;
    const uint32_t bar0 = base + OFF_BAR;
    auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
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
        tmem_alloc(base + OFF_TMEM_SLOT, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEM_SLOT);
    constexpr uint32_t STAGE16 = KV_BYTES >> 4;

    if (warp == WARP_TMA_K || warp == WARP_TMA_V) {
        // ------------------------------ TMA producers -----------------------------
        if (lane == 0 && n > 0) {
            const bool is_k = warp == WARP_TMA_K;
            const CUtensorMap* tm = is_k ? &tmk : &tmv;
            const int stages = is_k ? K_STAGES : V_STAGES;
            const int FULL = is_k ? K_FULL : V_FULL, EMPTY = is_k ? K_EMPTY : V_EMPTY;
            const uint32_t ring = is_k ? sK : sV;
            tma_prefetch_desc(tm);
            const uint64_t keep = l2_policy_evict_last();
            if (is_k) {
                tma_prefetch_desc(&tmq);
                mbar_arrive_expect_tx(bar(Q_FULL), Q_BYTES);
                tma_load_4d(sQ, &tmq, bar(Q_FULL), 0, h, q0, b);
                tma_load_4d(sQ + Q_HALF, &tmq, bar(Q_FULL), 64, h, q0, b);
            }
            int par[3] = {-1, -1, -1};                 // parity of the last copy issued per stage
            bool ok = true;
            for (int k = 0; k < nsteps && ok; ++k) {
                const int st = k % stages, use = (k / stages) & 1;
                const int key_a = block_of(2 * k) * BK, key_b = block_of(2 * k + 1) * BK;
                ok = wait_thread(bar(EMPTY + st), use ^ 1, wc);
                if (!ok) break;
                const uint32_t dst = ring + st * KV_BYTES;
                mbar_arrive_expect_tx(bar(FULL + st), KV_BYTES);
                tma_load_4d_hint(dst, tm, bar(FULL + st), 0, h, key_a, b, keep);
                tma_load_4d_hint(dst + BLOCK_BYTES, tm, bar(FULL + st), 0, h, key_b, b, keep);
                tma_load_4d_hint(dst + KV_DHALF, tm, bar(FULL + st), 64, h, key_a, b, keep);
                tma_load_4d_hint(dst + KV_DHALF + BLOCK_BYTES, tm, bar(FULL + st), 64, h, key_b, b, keep);
                par[st] = use;
            }
            if (!ok) {
                // let the copies already issued land before the CTA's shared memory goes away
                if (is_k) drain_wait(bar(Q_FULL), 0);
                for (int st = 0; st < stages; ++st)
                    if (par[st] >= 0) drain_wait(bar(FULL + st), par[st]);
            }
        }
    } else if (warp == WARP_QK) {
        // ------------------------------ Q K^T issuer ------------------------------
        if (lane == 0 && n > 0) {
            const uint32_t idesc_qk = make_idesc(1, 1, 1, 0, 0, BM, BN);
            const uint32_t hi = sdesc_hi();           // descriptors: common high half, low halves
            const uint32_t q_lo = sdesc_lo(sQ, 16), k_lo = sdesc_lo(sK, 16);
            static_assert(Q_HALF == KV_DHALF, "Q and K tiles share the offset of their second half of d");
            bool ok = wait_thread(bar(Q_FULL), 0, wc);
            for (int k = 0; k < nsteps && ok; ++k) {
                const int sb = k % NBUF, ks = k % K_STAGES;
                // S(k) overwrites the buffer P(k - 3) was read from
                if (k >= NBUF) ok = wait_thread(bar(PV_DONE + sb), ((k - NBUF) / NBUF) & 1, wc);
                if (ok) ok = wait_thread(bar(K_FULL + ks), (k / K_STAGES) & 1, wc);
                if (!ok) break;
                tc_fence_after();
                mma8_f16_ss<KV_DHALF / 16, 2>(tmem + static_cast<uint32_t>(sb * BN), q_lo, k_lo + ks * STAGE16, hi,
                                              idesc_qk, 0u);
                mma_commit(bar(S_FULL + sb));
                mma_commit(bar(K_EMPTY + ks));
            }
            mma_commit(bar(DRAIN_QK));
            drain_wait(bar(DRAIN_QK), 0);
        }
    } else if (warp == WARP_PV) {
        // -------------------------------- P V issuer ------------------------------
        if (lane == 0 && n > 0) {
            const uint32_t idesc_pv = make_idesc(1, 1, 1, 0, 1, BM, HD);
            const uint32_t hi = sdesc_hi();
            const uint32_t v_lo = sdesc_lo(sV, KV_DHALF);
            bool ok = true;
            for (int k = 0; k < nsteps && ok; ++k) {
                const int sb = k % NBUF, vs = k % V_STAGES;
                ok = wait_thread(bar(V_FULL + vs), (k / V_STAGES) & 1, wc);
                if (ok) ok = wait_thread(bar(P_FULL + sb), (k / NBUF) & 1, wc);
                if (!ok) break;
                tc_fence_after();
                // P: 8 columns per 16 keys; V: 2048 bytes per 16 keys, the second block 8 KB on
                mma8_f16_ts<32, BLOCK_BYTES / 16, 128>(tmem + T_O, tmem + static_cast<uint32_t>(sb * BN),
                                                       v_lo + vs * STAGE16, hi, idesc_pv, k > 0 ? 1u : 0u);
                mma_commit(bar(V_EMPTY + vs));
                mma_commit(bar(PV_DONE + sb));
                if (k + 1 == nsteps) mma_commit(bar(O_FINAL));
            }
            mma_commit(bar(DRAIN));
            drain_wait(bar(DRAIN), 0);
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
        // list entry i (0 past the list: the repeat of an odd list's last block)
        auto entry_of = [&](int i) { return i < n ? static_cast<unsigned>(list[i]) : 0u; };
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
            if (lim0 > 0 || lim1 > 0) {                   // warp-uniform
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
    if (p.kv_list) {
        if (configure_smem(reinterpret_cast<const void*>(sparse::pair::attn_fwd_sparse_pair_kernel),
                           sparse::pair::SMEM_BYTES) != 0)
            return -1;
        sparse::pair::attn_fwd_sparse_pair_kernel<<<grid, sparse::pair::NTHREADS, sparse::pair::SMEM_BYTES, stream>>>(
            tq, tk64, tv64, to, p);
        return cudaGetLastError() == cudaSuccess ? 0 : -1;
    }
    if (configure_smem(reinterpret_cast<const void*>(sparse::attn_fwd_sparse_kernel), sparse::SMEM_BYTES) != 0)
        return -1;
    sparse::attn_fwd_sparse_kernel<<<grid, sparse::NTHREADS, sparse::SMEM_BYTES, stream>>>(tq, tk64, tv64, to, p);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace wan
