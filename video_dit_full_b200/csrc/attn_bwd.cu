// bf16 backward of the Wan DiT full (non-causal) self-attention on sm_100a.
//
// The training step differentiates the same full spatio-temporal attention
// ("Wan 2.1 ... paper-podcast summary", section "先看现象": beta = 8 for the
// non-causal backward in the cost model).  With P = exp(S/sqrt(D) - lse),
// D_i = rowsum(dO_i * O_i) and dS = P * (dP - D):
//     dV = P^T dO,  dK = dS^T Q / sqrt(D),  dQ = dS K / sqrt(D),  dP = dO V^T.
//
// Three kernels:
//   bwd_prep    D_i = sum_d dO_id O_id (fp32) and zeroing of the fp32 dQ accumulator.
//   bwd_main    one CTA per 128-key tile of one (batch, head), eight gradient warps (two
//               threads per key row); K_j, V_j stay in
//               shared memory while the CTA walks every 128-row Q tile i:
//                 S^T = K Q_i^T, dP^T = V dO_i^T            (tcgen05, TMEM)
//                 P^T = exp2(S^T c - lse_i log2 e)          (softmax warpgroup)
//                 dV += P^T dO_i                            (A = P^T in TMEM)
//                 dS^T = P^T (dP^T - D_i)  -> TMEM and smem (into dO_i's buffer)
//                 dK += dS^T Q_i                            (A = dS^T in TMEM)
//                 dQ_i^T = K^T dS^T  -> TMEM (dP^T's columns, so the next tile's S^T can
//                                       start at once) -> shared (fp32) -> TMA reduce-add
//                                       into the accumulator (a dedicated reducer warp)
//               P is recomputed from the forward's LSE; nothing of size S x S is stored.
//   bwd_dq      dQ = bf16(accumulator / sqrt(D)).
//
// Queries and keys may differ in length (Sq, Skv): the block's cross-attention to the
// 512-token umT5 text embedding ("Wan 2.1 ... paper-podcast summary", section
// "干预与形式化").  With few key tiles (Skv = 512 gives 4 per head) one CTA per key tile
// would leave most SMs idle, so the caller may split each key tile's Q range over nsplit
// CTAs: each then adds its partial dK, dV into fp32 accumulators by TMA reduce-add (as dQ),
// and bwd_dq converts those too.  With nsplit = 1 each CTA writes its dK, dV tiles in bf16.
#include <cuda.h>

#include "sm100_ptx.cuh"
#include "wan_attn_internal.h"

namespace wan {
namespace bwd {

constexpr int BM = 128;                  // keys per CTA (and queries per Q tile)
constexpr int HD = 128;
constexpr int TILE_BYTES = BM * HD * 2;  // 32 KB bf16 tile
constexpr int HALF_BYTES = TILE_BYTES / 2;

constexpr int OFF_K = 0;
constexpr int OFF_V = OFF_K + TILE_BYTES;
// Two stages of [Q_i | dO_i] (64 KB each).  Within a tile, dS^T overwrites dO_i once dV is done;
// after the dK and dQ MMAs the whole stage holds the fp32 dQ^T tile [query][d] for the TMA reduce.
constexpr int OFF_STAGE = OFF_V + TILE_BYTES;
constexpr int STAGE_BYTES = 2 * TILE_BYTES;
constexpr int OFF_VEC = OFF_STAGE + 2 * STAGE_BYTES;   // per warp: 64 fp32 lse*log2(e), 64 fp32 D_i
constexpr int VEC_BYTES = 2 * 64 * 4;
constexpr int OFF_BAR = OFF_VEC + 8 * VEC_BYTES;
enum Bar { KV_FULL = 0, QDO_FULL = 1, QDO_EMPTY = 3, S_FULL = 5, DP_FULL = 6, P_READY = 7, DV_DONE = 8,
           DS_READY = 9, DQ_FULL = 10, DQ_DRAINED = 11, FINAL = 12, DRAIN = 13, STAGED = 14, DS_SMEM = 15,
           RED_DONE = 16, EPI_STAGED = 17, NBARS = 18 };
// split epilogue: dV (stage 0) and dK (stage 1) as four [128 key][32 d] fp32 sub-tiles each,
// 128-byte swizzled, one TMA reduce-add per sub-tile
constexpr int SUB_BYTES = BM * 32 * 4;
constexpr int OFF_TMEM_SLOT = OFF_BAR + NBARS * 8;
constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
constexpr int SMEM_USED = OFF_ABORT + 8;
constexpr int SMEM_BYTES = SMEM_USED + 1024;
// warps 0-7 gradients (two threads per key row: warps 0-3 take queries 0-63 of a tile,
// warps 4-7 queries 64-127), 8 TMA, 9 MMA, 10 dQ reducer
constexpr int NTHREADS = 352;
constexpr int WARP_TMA = 8, WARP_MMA = 9, WARP_RED = 10;
constexpr int G_THREADS = 256;
constexpr int G_WARPS = G_THREADS / 32;
#ifndef WAN_BWD_WARP_ARRIVE
#define WAN_BWD_WARP_ARRIVE 1         // the gradient warps' barriers count one arrival per warp
#endif
constexpr int G_ARRIVALS = WAN_BWD_WARP_ARRIVE ? G_WARPS : G_THREADS;
constexpr uint32_t TMEM_COLS = 512;      // S^T | dP^T | dV | dK
constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 384;
constexpr float LOG2E = 1.4426950408889634f;
#ifndef WAN_BWD_POLY_PAIRS
#define WAN_BWD_POLY_PAIRS 2          // of every 8 pairs of exponentials in P, this many use exp2_poly3
#endif
constexpr int BWD_POLY_PAIRS = WAN_BWD_POLY_PAIRS;

// A gradient warp's arrival on one of its barriers, after every lane's writes and fences: one
// arrival per warp (lane 0, once the warp has converged) or one per thread.
__device__ __forceinline__ void g_arrive(uint32_t bar, int lane) {
    if (WAN_BWD_WARP_ARRIVE) {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar);
    } else {
        mbar_arrive(bar);
    }
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 8 MMAs of K = 16 over a [128 rows][128 cols] bf16 tile pair, both K-major (K = the 128 columns).
// Shared-memory operands are given as their descriptors' low halves (lo_of: address and leading
// offset), `hi` the common high half.
__device__ __forceinline__ uint32_t lo_kmajor(uint32_t smem) { return sdesc_lo(smem, 16); }
__device__ __forceinline__ uint32_t lo_mnmajor(uint32_t smem) { return sdesc_lo(smem, HALF_BYTES); }
__device__ __forceinline__ void mma_kmajor(uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem, uint32_t hi,
                                           uint32_t idesc, bool accumulate) {
    mma8_f16_ss<HALF_BYTES / 16, 2>(d_tmem, lo_kmajor(a_smem), lo_kmajor(b_smem), hi, idesc, accumulate ? 1u : 0u);
}

// A in TMEM (bf16, 128 x 128), B MN-major in shared memory: K = the 128 rows of the B tile.
// A's columns for K = 0-63 start at a_tmem, those for K = 64-127 at a_tmem + 64 (each half of
// the row is written by its own thread into the TMEM columns it has just read).
__device__ __forceinline__ void mma_ts_bmn(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_smem, uint32_t hi,
                                           uint32_t idesc, bool accumulate) {
    mma8_f16_ts<64, 512, 128>(d_tmem, a_tmem, lo_mnmajor(b_smem), hi, idesc, accumulate ? 1u : 0u);
}

// A and B both MN-major in shared memory, K = the 128 rows of both tiles.
__device__ __forceinline__ void mma_ss_mn(uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem, uint32_t hi,
                                          uint32_t idesc) {
    mma8_f16_ss<512, 128>(d_tmem, lo_mnmajor(a_smem), lo_mnmajor(b_smem), hi, idesc, 0u);
}

__global__ void __launch_bounds__(NTHREADS, 1)
bwd_main_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmdo,
                const __grid_constant__ CUtensorMap tmdq, const __grid_constant__ CUtensorMap tmdk,
                const __grid_constant__ CUtensorMap tmdv, const BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_addr);

    const int warp = warp_id();
    const int lane = lane_id();
    const int h = blockIdx.y;
    const int b = blockIdx.z / p.nsplit, split = blockIdx.z % p.nsplit;
    const int kv0 = blockIdx.x * BM;
    const int Sq = p.Sq, Skv = p.Skv;
    // this CTA's Q tiles: [i_first, i_first + nq) of the (b, h)'s nq_all (nsplit <= nq_all)
    const int nq_all = (Sq + BM - 1) / BM;
    const int i_first = static_cast<int>(static_cast<long long>(split) * nq_all / p.nsplit);
    const int nq = static_cast<int>(static_cast<long long>(split + 1) * nq_all / p.nsplit) - i_first;

    const uint32_t sK = base + OFF_K, sV = base + OFF_V;
    auto sQ = [&](int s) { return base + OFF_STAGE + s * STAGE_BYTES; };
    auto sDO = [&](int s) { return base + OFF_STAGE + s * STAGE_BYTES + TILE_BYTES; };
    const uint32_t bar0 = base + OFF_BAR;
    auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
    const WaitCtl wc{abort_flag, p.wait_budget_ns, p.status};

    if (threadIdx.x == 0) {
        mbar_init(bar(KV_FULL), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(QDO_FULL + s), 1);
            mbar_init(bar(QDO_EMPTY + s), 2);    // the MMAs' commit + the dQ reducer's read-out
        }
        mbar_init(bar(S_FULL), 1);
        mbar_init(bar(DP_FULL), 1);
        mbar_init(bar(P_READY), G_ARRIVALS);
        mbar_init(bar(DV_DONE), 1);
        mbar_init(bar(DS_READY), G_ARRIVALS);     // dS^T in TMEM (dK may start)
        mbar_init(bar(DS_SMEM), G_ARRIVALS);      // dS^T in shared memory (dQ may start)
        mbar_init(bar(DQ_FULL), 1);
        mbar_init(bar(DQ_DRAINED), G_ARRIVALS);
        mbar_init(bar(FINAL), 1);
        mbar_init(bar(DRAIN), 1);
        mbar_init(bar(STAGED), G_ARRIVALS);
        mbar_init(bar(RED_DONE), 1);
        mbar_init(bar(EPI_STAGED), G_ARRIVALS);
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
            tma_prefetch_desc(&tmdo);
            mbar_arrive_expect_tx(bar(KV_FULL), 2 * TILE_BYTES);
            tma_load_4d(sK, &tmk, bar(KV_FULL), 0, h, kv0, b);
            tma_load_4d(sK + HALF_BYTES, &tmk, bar(KV_FULL), 64, h, kv0, b);
            tma_load_4d(sV, &tmv, bar(KV_FULL), 0, h, kv0, b);
            tma_load_4d(sV + HALF_BYTES, &tmv, bar(KV_FULL), 64, h, kv0, b);
            const uint64_t keep = l2_policy_evict_last();
            int par[2] = {-1, -1};
            bool ok = true;
            for (int i = 0; i < nq; ++i) {
                const int s = i & 1;
                const int use = (i >> 1) & 1;
                ok = wait_thread(bar(QDO_EMPTY + s), use ^ 1, wc);
                if (!ok) break;
                const uint32_t fb = bar(QDO_FULL + s);
                mbar_arrive_expect_tx(fb, 2 * TILE_BYTES);
                const int q_tok = (i_first + i) * BM;
                tma_load_4d_hint(sQ(s), &tmq, fb, 0, h, q_tok, b, keep);
                tma_load_4d_hint(sQ(s) + HALF_BYTES, &tmq, fb, 64, h, q_tok, b, keep);
                tma_load_4d_hint(sDO(s), &tmdo, fb, 0, h, q_tok, b, keep);
                tma_load_4d_hint(sDO(s) + HALF_BYTES, &tmdo, fb, 64, h, q_tok, b, keep);
                par[s] = use;
            }
            if (!ok) {
                drain_wait(bar(KV_FULL), 0);
                for (int s = 0; s < 2; ++s)
                    if (par[s] >= 0) drain_wait(bar(QDO_FULL + s), par[s]);
            }
        }
    } else if (warp == WARP_MMA) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0) {
            const uint32_t id_kk = make_idesc(1, 1, 1, 0, 0, BM, BM);   // both K-major
            const uint32_t id_tb = make_idesc(1, 1, 1, 0, 1, BM, HD);   // A in TMEM, B MN-major
            const uint32_t id_mm = make_idesc(1, 1, 1, 1, 1, HD, BM);   // both MN-major
            const uint32_t hi = sdesc_hi();
            bool ok = wait_thread(bar(KV_FULL), 0, wc);
            if (ok) ok = wait_thread(bar(QDO_FULL + 0), 0, wc);
            if (ok) {
                tc_fence_after();
                mma_kmajor(tmem + T_S, sK, sQ(0), hi, id_kk, false);      // S^T = K Q^T of the first tile
                mma_commit(bar(S_FULL));
                mma_kmajor(tmem + T_DP, sV, sDO(0), hi, id_kk, false);    // dP^T = V dO^T
                mma_commit(bar(DP_FULL));
            }
            for (int i = 0; i < nq && ok; ++i) {
                const int s = i & 1;
                const uint32_t q_s = sQ(s), do_s = sDO(s);
                ok = wait_thread(bar(P_READY), i & 1, wc);
                if (!ok) break;
                tc_fence_after();
                mma_ts_bmn(tmem + T_DV, tmem + T_S, do_s, hi, id_tb, i > 0);   // dV += P^T dO
                mma_commit(bar(DV_DONE));
                ok = wait_thread(bar(DS_READY), i & 1, wc);
                if (!ok) break;
                tc_fence_after();
                mma_ts_bmn(tmem + T_DK, tmem + T_DP, q_s, hi, id_tb, i > 0);   // dK += dS^T Q
                ok = wait_thread(bar(DS_SMEM), i & 1, wc);
                if (!ok) break;
                // dQ^T = K^T dS^T (dS^T in dO's buffer) into dP^T's columns, which the dK MMA just
                // read: S^T's columns are free for the next tile at once
                mma_ss_mn(tmem + T_DP, sK, do_s, hi, id_mm);
                mma_commit(bar(DQ_FULL));
                mma_commit(bar(QDO_EMPTY + s));
                if (i + 1 < nq) {
                    // the next tile's S^T runs while the gradient warps copy dQ^T out; its dP^T
                    // (needed only after its P) once that copy has freed the columns
                    const int s1 = (i + 1) & 1;
                    ok = wait_thread(bar(QDO_FULL + s1), ((i + 1) >> 1) & 1, wc);
                    if (!ok) break;
                    tc_fence_after();
                    mma_kmajor(tmem + T_S, sK, sQ(s1), hi, id_kk, false);
                    mma_commit(bar(S_FULL));
                    ok = wait_thread(bar(DQ_DRAINED), i & 1, wc);
                    if (!ok) break;
                    tc_fence_after();
                    mma_kmajor(tmem + T_DP, sV, sDO(s1), hi, id_kk, false);
                    mma_commit(bar(DP_FULL));
                }
            }
            if (ok) mma_commit(bar(FINAL));
            mma_commit(bar(DRAIN));
            drain_wait(bar(DRAIN), 0);
        }
    } else if (warp == WARP_RED) {
        // ------------------ dQ reducer: TMA reduce-add of each dQ tile ------------
        if (lane == 0) {
            bool ok = true;
            for (int i = 0; i < nq && ok; ++i) {
                ok = wait_thread(bar(STAGED), i & 1, wc);
                if (!ok) break;
                tma_reduce_add_4d(&tmdq, base + OFF_STAGE + (i & 1) * STAGE_BYTES, 0, h, (i_first + i) * BM, b);
                bulk_commit_group();
                bulk_wait_read_all();                         // the stage may be refilled now
                mbar_arrive(bar(QDO_EMPTY + (i & 1)));
            }
            bulk_wait_all();
            if (p.nsplit > 1 && ok) {
                // split Q range: add this CTA's dV and dK tiles into the fp32 accumulators
                mbar_arrive(bar(RED_DONE));                   // the stages are free for them
                ok = wait_thread(bar(EPI_STAGED), 0, wc);
                if (ok) {
                    for (int which = 0; which < 2; ++which)
                        for (int st = 0; st < 4; ++st)
                            tma_reduce_add_4d(which ? &tmdk : &tmdv,
                                              base + OFF_STAGE + which * STAGE_BYTES + st * SUB_BYTES, st * 32, h,
                                              kv0, b);
                    bulk_commit_group();
                    bulk_wait_all();
                }
            }
        }
    } else {
        // -------- gradient warps: two threads per key row (or per d for dQ^T) -------
        // Thread (j, hq): key row / TMEM lane j = 32*(warp%4) + lane; query half hq = warp/4
        // covers queries 64hq..64hq+63 of each Q tile.  It writes P^T and dS^T (bf16) into the
        // first 32 of the 64 TMEM columns it has just read, so the halves never race.
        const int hq = warp >> 2;
        const int cb = hq * 64;                            // first query column of this half
        const int j = (warp & 3) * 32 + lane;              // 0..127
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + T_S + lane_off + cb, tDP = tmem + T_DP + lane_off + cb;
        const int key = kv0 + j;
        const bool key_ok = key < Skv;
        const float c = p.scale_log2;
        const size_t bh = static_cast<size_t>(b) * p.H + h;
        // each warp keeps its own copy of its 64 queries' lse / D (no cross-warp barrier needed)
        float* s_lse = reinterpret_cast<float*>(smem + OFF_VEC + warp * VEC_BYTES);
        float* s_del = s_lse + 64;
        bool ok = true;
        // a tile's lse / D come from global memory one tile ahead, so their latency hides
        // behind the previous tile instead of delaying the wait for S^T
        float nl[2], nd[2];
        auto load_vec = [&](int ti) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int qi = (i_first + ti) * BM + cb + e * 32 + lane;
                nl[e] = qi < Sq ? p.lse[bh * Sq + qi] * LOG2E : INFINITY;
                nd[e] = qi < Sq ? p.delta[bh * Sq + qi] : 0.f;
            }
        };
        if (nq > 0) load_vec(0);
        for (int i = 0; i < nq && ok; ++i) {
            __syncwarp();                                    // previous tile's values no longer read
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                s_lse[e * 32 + lane] = nl[e];
                s_del[e * 32 + lane] = nd[e];
            }
            __syncwarp();
            if (i + 1 < nq) load_vec(i + 1);

            ok = wait_warp(bar(S_FULL), i & 1, wc);
            if (!ok) break;
            tc_fence_after();
            float pr[64];
            {
                uint32_t* sr = reinterpret_cast<uint32_t*>(pr);
                tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                tmem_wait_ld();
            }
#pragma unroll
            for (int e = 0; e < 64; ++e) {
                // a share of the exponentials runs on the FMA pipe (the MUFU bounds this phase)
                const float x = fmaf(pr[e], c, -s_lse[e]);
                const float pe = ((e >> 1) & 7) < BWD_POLY_PAIRS ? exp2_poly3(x) : ex2_approx(x);
                pr[e] = key_ok ? pe : 0.f;
            }
            {
                uint32_t pk[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) pk[e] = pack_bf16x2(pr[2 * e], pr[2 * e + 1]);
                tmem_st32(tS, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            g_arrive(bar(P_READY), lane);

            ok = wait_warp(bar(DP_FULL), i & 1, wc);
            if (!ok) break;
            tc_fence_after();
            uint32_t dsp[32];                                // this half-row's dS^T, bf16 pairs
            {
                uint32_t dp[64];
                tmem_ld32(tDP, *reinterpret_cast<uint32_t(*)[32]>(&dp[0]));
                tmem_ld32(tDP + 32, *reinterpret_cast<uint32_t(*)[32]>(&dp[32]));
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    // dS = P (dP - D), a pair at a time
                    const float2 dd = fsub2(make_float2(__uint_as_float(dp[2 * e]), __uint_as_float(dp[2 * e + 1])),
                                            make_float2(s_del[2 * e], s_del[2 * e + 1]));
                    const float2 ds = fmul2(make_float2(pr[2 * e], pr[2 * e + 1]), dd);
                    dsp[e] = pack_bf16x2(ds.x, ds.y);
                }
            }
            tmem_st32(tDP, dsp);
            tmem_wait_st();
            tc_fence_before();
            g_arrive(bar(DS_READY), lane);
            // dS^T row j, queries cb..cb+63 -> the 128-byte swizzled row j of half hq, in dO's
            // buffer: only once dV (the last reader of dO) is done
            ok = wait_warp(bar(DV_DONE), i & 1, wc);
            if (!ok) break;
            uint8_t* half_row = smem + OFF_STAGE + (i & 1) * STAGE_BYTES + TILE_BYTES + hq * HALF_BYTES + j * 128;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
                *reinterpret_cast<uint4*>(half_row + ((ch ^ (j & 7)) * 16)) =
                    make_uint4(dsp[4 * ch], dsp[4 * ch + 1], dsp[4 * ch + 2], dsp[4 * ch + 3]);
            fence_async_smem();
            g_arrive(bar(DS_SMEM), lane);

            ok = wait_warp(bar(DQ_FULL), i & 1, wc);
            if (!ok) break;
            tc_fence_after();
            // dQ^T: TMEM lane = d (= j), column = query.  Copy queries cb..cb+63 into the stage as
            // fp32 [query][d] (its Q and dS^T are consumed), free the TMEM columns, and let the
            // reducer warp add the tile into the accumulator by TMA.
            float* stage = reinterpret_cast<float*>(smem + OFF_STAGE + (i & 1) * STAGE_BYTES);
#pragma unroll 1
            for (int q = 0; q < 2; ++q) {
                uint32_t v[32];
                tmem_ld32(tDP + q * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) stage[(cb + q * 32 + e) * HD + j] = __uint_as_float(v[e]);
            }
            tc_fence_before();
            g_arrive(bar(DQ_DRAINED), lane);
            fence_async_smem();
            g_arrive(bar(STAGED), lane);
        }
        if (ok) ok = wait_warp(bar(FINAL), 0, wc);
        if (ok && p.nsplit > 1) {
            // stage dV, dK (fp32, unscaled) for the reducer warp's TMA reduce-adds, once it has
            // finished reading the stages for dQ
            ok = wait_warp(bar(RED_DONE), 0, wc);
            if (ok) {
                tc_fence_after();
#pragma unroll 1
                for (int which = 0; which < 2; ++which) {
                    const uint32_t src = tmem + (which ? T_DK : T_DV) + lane_off + cb;
#pragma unroll 1
                    for (int q = 0; q < 2; ++q) {
                        uint32_t v[32];
                        tmem_ld32(src + q * 32, v);
                        tmem_wait_ld();
                        // sub-tile hq*2+q holds d = 32(hq*2+q) .. +31; row j, 16-byte chunk c at c ^ (j % 8)
                        uint8_t* row = smem + OFF_STAGE + which * STAGE_BYTES + (hq * 2 + q) * SUB_BYTES + j * 128;
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch)
                            *reinterpret_cast<uint4*>(row + ((ch ^ (j & 7)) * 16)) =
                                make_uint4(v[4 * ch], v[4 * ch + 1], v[4 * ch + 2], v[4 * ch + 3]);
                    }
                }
                fence_async_smem();
                g_arrive(bar(EPI_STAGED), lane);
            }
        } else if (ok) {
            tc_fence_after();
            const size_t row = ((static_cast<size_t>(b) * Skv + key) * p.H + h) * HD + cb;
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {
                const uint32_t src = tmem + (which ? T_DK : T_DV) + lane_off + cb;
                const float mul = which ? p.scale : 1.f;
                __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(which ? p.dk : p.dv) + row;
#pragma unroll 1
                for (int q = 0; q < 2; ++q) {
                    uint32_t v[32];
                    tmem_ld32(src + q * 32, v);
                    tmem_wait_ld();
                    uint4 pk[4];
                    uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pw[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * mul, __uint_as_float(v[2 * e + 1]) * mul);
                    if (key_ok) {
                        uint4* d4 = reinterpret_cast<uint4*>(dst + q * 32);
#pragma unroll
                        for (int e = 0; e < 4; ++e) d4[e] = pk[e];
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == WARP_MMA) tmem_dealloc(tmem, TMEM_COLS);
}

// D_i = sum_d dO_id * O_id (fp32) for every (b, s, h) row, and dQ accumulator := 0.
// 16 threads per row, 8 elements (16 bytes) each.
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ dout,
                                                       float* __restrict__ delta, float* __restrict__ dq_acc,
                                                       long long rows, int S, int H) {
    const long long total = rows * 16;
    const int lane = threadIdx.x & 31;
    const long long warp0 = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x - lane;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long t0 = warp0; t0 < total; t0 += stride) {        // warp-uniform trip count
        const long long t = t0 + lane;
        const bool valid = t < total;
        const long long r = t >> 4;               // row index over [B, S, H]
        const int part = static_cast<int>(t & 15);
        float acc = 0.f;
        if (valid) {
            const uint4 ov = *reinterpret_cast<const uint4*>(o + r * HD + part * 8);
            const uint4 dv = *reinterpret_cast<const uint4*>(dout + r * HD + part * 8);
            const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
            const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 a = __bfloat1622float2(o2[e]);
                const float2 c = __bfloat1622float2(d2[e]);
                acc = fmaf(a.x, c.x, acc);
                acc = fmaf(a.y, c.y, acc);
            }
        }
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (valid) {
            float4* z = reinterpret_cast<float4*>(dq_acc + r * HD + part * 8);
            z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
            z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (part == 0) {
                const long long h = r % H;
                const long long bs = r / H;
                const long long s = bs % S;
                const long long b = bs / S;
                delta[(b * H + h) * S + s] = acc;
            }
        }
    }
}

// dQ = bf16(acc * scale), 8 elements per thread.
__global__ void __launch_bounds__(256) bwd_dq_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq,
                                                     long long n8, float scale) {
    const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long t = tid; t < n8; t += stride) {
        const float4 a = reinterpret_cast<const float4*>(acc)[2 * t];
        const float4 c = reinterpret_cast<const float4*>(acc)[2 * t + 1];
        uint4 out;
        out.x = pack_bf16x2(a.x * scale, a.y * scale);
        out.y = pack_bf16x2(a.z * scale, a.w * scale);
        out.z = pack_bf16x2(c.x * scale, c.y * scale);
        out.w = pack_bf16x2(c.z * scale, c.w * scale);
        reinterpret_cast<uint4*>(dq)[t] = out;
    }
}

}  // namespace bwd

int launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
               const CUtensorMap& tdq, const CUtensorMap& tdk, const CUtensorMap& tdv, BwdParams p,
               bool allow_split, const void* o, const void* dout, void* dq, cudaStream_t stream) {
    const long long rows = static_cast<long long>(p.B) * p.Sq * p.H;
    const long long kv_rows = static_cast<long long>(p.B) * p.Skv * p.H;
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // Split each key tile's Q range when the key tiles alone give fewer than 4 waves of CTAs:
    // then aim at >= 8 waves (whole waves matter less as the count grows).
    const int nkv = (p.Skv + bwd::BM - 1) / bwd::BM;
    const int nq_all = (p.Sq + bwd::BM - 1) / bwd::BM;
    const long long ctas = static_cast<long long>(nkv) * p.H * p.B;
    int ns = 1;
    if (allow_split && ctas < 4LL * sms) {
        ns = static_cast<int>((8LL * sms + ctas - 1) / ctas);
        if (ns > nq_all) ns = nq_all;
        while (ns > 1 && static_cast<long long>(p.B) * ns > 65535) --ns;
    }
    p.nsplit = ns;
    const int ew_blocks = sms * 8;     // grid-stride elementwise kernels: 8 blocks of 256 per SM
    bwd::bwd_prep_kernel<<<ew_blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(o),
                                                        static_cast<const __nv_bfloat16*>(dout), p.delta, p.dq_acc,
                                                        rows, p.Sq, p.H);
    if (cudaGetLastError() != cudaSuccess) return -1;
    if (ns > 1) {
        const size_t acc_bytes = static_cast<size_t>(kv_rows) * bwd::HD * 4;
        if (cudaMemsetAsync(p.dk_acc, 0, acc_bytes, stream) != cudaSuccess ||
            cudaMemsetAsync(p.dv_acc, 0, acc_bytes, stream) != cudaSuccess)
            return -1;
    }
    if (configure_smem(reinterpret_cast<const void*>(bwd::bwd_main_kernel), bwd::SMEM_BYTES) != 0) return -1;
    const dim3 grid(nkv, p.H, p.B * ns);
    bwd::bwd_main_kernel<<<grid, bwd::NTHREADS, bwd::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, tdq, tdk, tdv, p);
    if (cudaGetLastError() != cudaSuccess) return -1;
    bwd::bwd_dq_kernel<<<ew_blocks, 256, 0, stream>>>(p.dq_acc, static_cast<__nv_bfloat16*>(dq), rows * 16,
                                                      p.scale);
    if (ns > 1) {
        bwd::bwd_dq_kernel<<<ew_blocks, 256, 0, stream>>>(p.dk_acc, static_cast<__nv_bfloat16*>(p.dk), kv_rows * 16,
                                                          p.scale);
        bwd::bwd_dq_kernel<<<ew_blocks, 256, 0, stream>>>(p.dv_acc, static_cast<__nv_bfloat16*>(p.dv), kv_rows * 16,
                                                          1.0f);
    }
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace wan
