// Thin inline-PTX wrappers for the sm_100a features the attention kernels use:
// mbarriers, TMA tensor loads, tcgen05 (TMEM alloc/ld/st, MMA, commit) and
// bounded waits that report a timeout instead of spinning for ever.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace wan {

// ----------------------------------------------------------------------------
// status codes a kernel can leave in the library's device status word
// ----------------------------------------------------------------------------
enum : int { kStatusOk = 0, kStatusTimeout = 4 };

__device__ __forceinline__ void report_status(int* status, int code) {
    atomicCAS(status, 0, code);
}

// ----------------------------------------------------------------------------
// shared-memory addresses and mbarriers
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Control block for bounded waits: a CTA-wide abort flag in shared memory and
// a time budget.  A wait that runs out of time sets the flag and the device
// status word; every other wait of the CTA then gives up at its next check.
// A wait that has already lasted kStatusPollNs (no healthy wait comes near it)
// also gives up when the device status word holds an error: once one CTA has
// timed out, the CTAs still to come do not each spend a whole budget.
struct WaitCtl {
    volatile int* abort_flag;   // shared memory
    uint64_t budget_ns;
    int* status;                // device status word of the library (global memory)
};

constexpr uint64_t kStatusPollNs = 1000000ull;   // 1 ms

__device__ __forceinline__ bool wait_expired(const WaitCtl& w, uint64_t t0) {
    if (*w.abort_flag) return true;
    const uint64_t waited = global_timer_ns() - t0;
    if (waited > w.budget_ns) {
        *w.abort_flag = 1;
        report_status(w.status, kStatusTimeout);
        return true;
    }
    if (waited > kStatusPollNs && w.budget_ns > kStatusPollNs && *reinterpret_cast<volatile int*>(w.status) != 0) {
        *w.abort_flag = 1;
        return true;
    }
    return false;
}

// Used only after an abort, to let the copies and MMAs a thread already issued
// land before the CTA's shared and tensor memory go away.  It ignores the abort
// flag and uses its own budget (those operations finish in microseconds; the
// budget only bounds a GPU that has stopped making progress), so a tiny
// user-set wait budget cannot cut it short.
constexpr uint64_t kDrainBudgetNs = 50000000ull;   // 50 ms
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > kDrainBudgetNs) break;
    }
}

// One thread waits for the phase of `bar` with the given parity.  false = gave up.
__device__ __forceinline__ bool wait_thread(uint32_t bar, uint32_t parity, const WaitCtl& w) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 0 && wait_expired(w, t0)) return false;
    }
}

// All 32 lanes of a warp wait; the result is the same on every lane.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, const WaitCtl& w) {
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        const bool done = mbar_try_wait(bar, parity);
        if (__all_sync(0xffffffffu, done)) return true;
        if ((it & 15u) == 15u) {
            int stop = 0;
            if ((threadIdx.x & 31) == 0) {
                if (t0 == 0) t0 = global_timer_ns();
                stop = wait_expired(w, t0) ? 1 : 0;
            }
            if (__shfl_sync(0xffffffffu, stop, 0)) return false;
        }
    }
}

// ----------------------------------------------------------------------------
// TMA
// ----------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// 4-D tiled load global -> shared, completion counted on `bar` (bytes).
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const void* tmap, uint32_t bar, int c0, int c1,
                                            int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// 2-D tiled load global -> shared.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, uint32_t bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

// 3-D tiled load global -> shared.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, uint32_t bar, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// Same, with an L2 cache policy (e.g. evict-last for tiles many CTAs re-read).
__device__ __forceinline__ void tma_load_4d_hint(uint32_t dst, const void* tmap, uint32_t bar, int c0, int c1,
                                                 int c2, int c3, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "l"(policy)
        : "memory");
}

// 4-D tiled reduce-add shared -> global (fp32 add into the tensor map's memory),
// tracked by the issuing thread's bulk async-group.
__device__ __forceinline__ void tma_reduce_add_4d(const void* tmap, uint32_t src, int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group"
        " [%0, {%2, %3, %4, %5}], [%1];" ::"l"(reinterpret_cast<uint64_t>(tmap)),
        "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
// 4-D tiled store shared -> global, tracked by the issuing thread's bulk async-group.  Parts of
// the box outside the tensor (rows past S) are not written.  The coordinates must be >= 0.
__device__ __forceinline__ void tma_store_4d(const void* tmap, uint32_t src, int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group"
        " [%0, {%2, %3, %4, %5}], [%1];" ::"l"(reinterpret_cast<uint64_t>(tmap)),
        "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
// Make this thread's ordinary shared-memory writes visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Barrier among `nthreads` threads (a multiple of 32) of the CTA on hardware barrier `id` (1-15).
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// 16-byte shared-memory store.
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}
// Address of 16-byte chunk `c` (0-7) of row `r` in a [rows][128 bytes] tile at `tile` (1024-byte
// aligned) laid out with the 128-byte swizzle that TMA uses: the chunk index is XORed with r % 8.
__device__ __forceinline__ uint32_t sw128_chunk(uint32_t tile, int r, int c) {
    return tile + static_cast<uint32_t>(r) * 128u + (static_cast<uint32_t>((c ^ r) & 7) << 4);
}

// A row's 64 bf16 (32 packed words) into its 128-byte row of a swizzled tile.
__device__ __forceinline__ void st_row_sw128(uint32_t tile, int r, const uint32_t (&w)[32]) {
#pragma unroll
    for (int c = 0; c < 8; ++c) st_shared_v4(sw128_chunk(tile, r, c), w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
}

__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the shared-memory sources of every committed bulk group have been read.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Wait until every committed bulk group has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// ----------------------------------------------------------------------------
// tcgen05: tensor memory
// ----------------------------------------------------------------------------
// Whole warp: allocate `ncols` TMEM columns; the base address lands in shared memory at dst.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: lane i of the warp gets row (lane base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// ----------------------------------------------------------------------------
// tcgen05: MMA
// ----------------------------------------------------------------------------
// Shared-memory matrix descriptor (sm_100 format): start address, leading and
// stride byte offsets (16-byte units), version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;   // descriptor version for sm_100
    d |= static_cast<uint64_t>(2) << 61;   // SWIZZLE_128B
    return d;
}

// Instruction descriptor for dense kind::f16 / kind::i8 / kind::f8f6f4 MMAs.
// dfmt: 0 f16, 1 f32, 2 s32.  afmt/bfmt: kind::f16 -> 0 f16, 1 bf16; kind::i8 -> 1 signed;
// kind::f8f6f4 -> 0 e4m3.  a_mn / b_mn: 1 if that operand is MN-major in shared memory.
__host__ __device__ constexpr uint32_t make_idesc(uint32_t dfmt, uint32_t afmt, uint32_t bfmt, uint32_t a_mn,
                                                  uint32_t b_mn, uint32_t M, uint32_t N) {
    return (dfmt << 4) | (afmt << 7) | (bfmt << 10) | (a_mn << 15) | (b_mn << 16) | ((N >> 3) << 17) |
           ((M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void mma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem], kind::f16.
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// kind::i8 (int8 inputs, int32 accumulate), both operands in shared memory.
__device__ __forceinline__ void mma_i8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// kind::f8f6f4 with A in tensor memory (e4m3 inputs, fp32 accumulate).
__device__ __forceinline__ void mma_f8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// kind::f8f6f4, both operands in shared memory.
__device__ __forceinline__ void mma_f8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every tcgen05 op this thread issued before has completed.
// The 8 MMAs of a K = 128 contraction (K = 16 each) in one asm block, A and B from shared memory.
// Step k reads A and B at (k / 4) * OFF_HI + (k % 4) * OFF_LO past their base descriptors, in
// the descriptors' 16-byte address units: K-major 128-byte-swizzled operands whose 64-wide halves
// of K lie h bytes apart take (h / 16, 2); MN-major ones with 2048 bytes per 16 rows of K take
// (512, 128).  a_lo / b_lo are the base descriptors' low halves (address and leading offset),
// `hi` their common high half (stride offset, version, swizzle): adding to the low half moves the
// start address, with no carry out of its 14-bit field while addresses stay below 256 KB.  The
// first MMA overwrites D unless `accumulate`; the others accumulate.
template <uint32_t OFF_HI, uint32_t OFF_LO>
__device__ __forceinline__ void mma8_f16_ss(uint32_t d, uint32_t a_lo, uint32_t b_lo, uint32_t hi, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p0, p1;\n\t.reg .b32 x, y;\n\t.reg .b64 a, b;\n\t"
        "setp.ne.b32 p0, %5, 0;\n\tsetp.eq.b32 p1, %4, %4;\n\t"
        "mov.b64 a, {%1, %3};\n\tmov.b64 b, {%2, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, p0;\n\t"
        "add.u32 x, %1, %6;\n\tadd.u32 y, %2, %6;\n\tmov.b64 a, {x, %3};\n\tmov.b64 b, {y, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, p1;\n\t"
        "add.u32 x, %1, %7;\n\tadd.u32 y, %2, %7;\n\tmov.b64 a, {x, %3};\n\tmov.b64 b, {y, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, p1;\n\t"
        "add.u32 x, %1, %8;\n\tadd.u32 y, %2, %8;\n\tmov.b64 a, {x, %3};\n\tmov.b64 b, {y, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, p1;\n\t"
        "add.u32 x, %1, %9;\n\tadd.u32 y, %2, %9;\n\tmov.b64 a, {x, %3};\n\tmov.b64 b, {y, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, p1;\n\t"
        "add.u32 x, %1, %10;\n\tadd.u32 y, %2, %10;\n\tmov.b64 a, {x, %3};\n\tmov.b64 b, {y, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, p1;\n\t"
        "add.u32 x, %1, %11;\n\tadd.u32 y, %2, %11;\n\tmov.b64 a, {x, %3};\n\tmov.b64 b, {y, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, p1;\n\t"
        "add.u32 x, %1, %12;\n\tadd.u32 y, %2, %12;\n\tmov.b64 a, {x, %3};\n\tmov.b64 b, {y, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, p1;\n\t}" ::"r"(d),
        "r"(a_lo), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate), "n"(OFF_LO), "n"(2 * OFF_LO),
        "n"(3 * OFF_LO), "n"(OFF_HI), "n"(OFF_HI + OFF_LO), "n"(OFF_HI + 2 * OFF_LO), "n"(OFF_HI + 3 * OFF_LO)
        : "memory");
}
// The 8 MMAs of a K = 128 contraction with A from TMEM (bf16 pairs, 8 columns per 16 elements of
// K): step k reads A at column a_tmem + (k / 4) * A_HI + (k % 4) * 8 and B at (k / 4) * B_HI +
// (k % 4) * B_LO past its base descriptor (low half b_lo, high half hi), as mma8_f16_ss.
template <uint32_t A_HI, uint32_t B_HI, uint32_t B_LO>
__device__ __forceinline__ void mma8_f16_ts(uint32_t d, uint32_t a_tmem, uint32_t b_lo, uint32_t hi, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p0, p1;\n\t.reg .b32 x, t;\n\t.reg .b64 b;\n\t"
        "setp.ne.b32 p0, %5, 0;\n\tsetp.eq.b32 p1, %4, %4;\n\t"
        "mov.b64 b, {%2, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], b, %4, p0;\n\t"
        "add.u32 x, %2, %6;\n\tadd.u32 t, %1, 8;\n\tmov.b64 b, {x, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, p1;\n\t"
        "add.u32 x, %2, %7;\n\tadd.u32 t, %1, 16;\n\tmov.b64 b, {x, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, p1;\n\t"
        "add.u32 x, %2, %8;\n\tadd.u32 t, %1, 24;\n\tmov.b64 b, {x, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, p1;\n\t"
        "add.u32 x, %2, %9;\n\tadd.u32 t, %1, %13;\n\tmov.b64 b, {x, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, p1;\n\t"
        "add.u32 x, %2, %10;\n\tadd.u32 t, %1, %14;\n\tmov.b64 b, {x, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, p1;\n\t"
        "add.u32 x, %2, %11;\n\tadd.u32 t, %1, %15;\n\tmov.b64 b, {x, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, p1;\n\t"
        "add.u32 x, %2, %12;\n\tadd.u32 t, %1, %16;\n\tmov.b64 b, {x, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, p1;\n\t}" ::"r"(d),
        "r"(a_tmem), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate), "n"(B_LO), "n"(2 * B_LO), "n"(3 * B_LO),
        "n"(B_HI), "n"(B_HI + B_LO), "n"(B_HI + 2 * B_LO), "n"(B_HI + 3 * B_LO), "n"(A_HI), "n"(A_HI + 8),
        "n"(A_HI + 16), "n"(A_HI + 24)
        : "memory");
}
// The 4 MMAs of an int8 K = 128 contraction (K = 32 each) in one asm block, A and B K-major with
// 128-byte rows in shared memory: step k reads both at k * 32 bytes past the base descriptors
// (low halves a_lo / b_lo, common high half hi).  The first MMA overwrites D.
__device__ __forceinline__ void mma4_i8_ss(uint32_t d, uint32_t a_lo, uint32_t b_lo, uint32_t hi, uint32_t idesc) {
    asm volatile(
        "{\n\t.reg .pred p0, p1;\n\t.reg .b32 x, y;\n\t.reg .b64 a, b;\n\t"
        "setp.ne.b32 p0, %4, %4;\n\tsetp.eq.b32 p1, %4, %4;\n\t"
        "mov.b64 a, {%1, %3};\n\tmov.b64 b, {%2, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], a, b, %4, p0;\n\t"
        "add.u32 x, %1, 2;\n\tadd.u32 y, %2, 2;\n\tmov.b64 a, {x, %3};\n\tmov.b64 b, {y, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], a, b, %4, p1;\n\t"
        "add.u32 x, %1, 4;\n\tadd.u32 y, %2, 4;\n\tmov.b64 a, {x, %3};\n\tmov.b64 b, {y, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], a, b, %4, p1;\n\t"
        "add.u32 x, %1, 6;\n\tadd.u32 y, %2, 6;\n\tmov.b64 a, {x, %3};\n\tmov.b64 b, {y, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], a, b, %4, p1;\n\t}" ::"r"(d),
        "r"(a_lo), "r"(b_lo), "r"(hi), "r"(idesc)
        : "memory");
}
// The 2 MMAs of an e4m3 K = 64 contraction (K = 32 each) with A from TMEM (a_tmem, a_tmem + 8)
// and B MN-major in shared memory, 4096 bytes per 32 rows of K (base descriptor low half b_lo,
// high half hi).  The first MMA accumulates only if `accumulate`.
__device__ __forceinline__ void mma2_f8_ts(uint32_t d, uint32_t a_tmem, uint32_t b_lo, uint32_t hi, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p0, p1;\n\t.reg .b32 x, t;\n\t.reg .b64 b;\n\t"
        "setp.ne.b32 p0, %5, 0;\n\tsetp.eq.b32 p1, %4, %4;\n\t"
        "mov.b64 b, {%2, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], b, %4, p0;\n\t"
        "add.u32 x, %2, 256;\n\tadd.u32 t, %1, 8;\n\tmov.b64 b, {x, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [t], b, %4, p1;\n\t}" ::"r"(d),
        "r"(a_tmem), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Low and high halves of a shared-memory descriptor (sdesc_sw128).
__device__ __forceinline__ uint32_t sdesc_lo(uint32_t saddr, uint32_t lbo_bytes) {
    return static_cast<uint32_t>(sdesc_sw128(saddr, lbo_bytes, 1024));
}
__device__ __forceinline__ uint32_t sdesc_hi() { return static_cast<uint32_t>(sdesc_sw128(0, 16, 1024) >> 32); }

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// ----------------------------------------------------------------------------
// math helpers
// ----------------------------------------------------------------------------
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x on the FMA and integer pipes instead of the MUFU: x = n + f with n the
// nearest integer (adding 1.5 * 2^23 rounds x into the low mantissa bits) and
// f in [-1/2, 1/2]; 2^f from a degree-3 polynomial fitted for minimax relative
// error by video_dit_full_b200/fit_exp2_poly.py (max relative error 7.5e-5,
// far below bf16's 2^-9); 2^n is added to the exponent field.  x is clamped to
// -125 so the result stays a normal float (an input of -inf gives 2^-125.5).
__device__ __forceinline__ float exp2_poly3(float x) {
    x = fmaxf(x, -125.f);
    const float j = x + 12582912.f;
    const float f = x - (j - 12582912.f);
    float p = fmaf(0.05517149344086647f, f, 0.24261093139648438f);
    p = fmaf(p, f, 0.6932609677314758f);
    p = fmaf(p, f, 0.9999280571937561f);
    return __int_as_float(__float_as_int(p) + (__float_as_int(j) << 23));
}

// Packed fp32 pairs (sm_100): two FMAs / adds in one instruction.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
// Three-input maximum (sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// exp2_poly3 for a pair in packed arithmetic: the same clamp, range split, coefficients and
// exponent-field add per element, so each result equals exp2_poly3 of its input.
__device__ __forceinline__ float2 exp2_poly3_x2(float2 x) {
    x = make_float2(fmaxf(x.x, -125.f), fmaxf(x.y, -125.f));
    const float2 magic = make_float2(12582912.f, 12582912.f);
    const float2 j = fadd2(x, magic);                       // n in the low mantissa bits
    const float2 f = fsub2(x, fsub2(j, magic));             // exact: x - n
    float2 p = ffma2(make_float2(0.05517149344086647f, 0.05517149344086647f), f,
                     make_float2(0.24261093139648438f, 0.24261093139648438f));
    p = ffma2(p, f, make_float2(0.6932609677314758f, 0.6932609677314758f));
    p = ffma2(p, f, make_float2(0.9999280571937561f, 0.9999280571937561f));
    return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(j.x) << 23)),
                       __int_as_float(__float_as_int(p.y) + (__float_as_int(j.y) << 23)));
}

// 2^x for a pair, for results that are rounded to e4m3 next (3 mantissa bits): the same
// range split as exp2_poly3 with a degree-2 minimax polynomial from
// video_dit_full_b200/fit_exp2_poly.py --degree 2 (max relative error 1.73e-3, a
// thirty-sixth of e4m3's half step), in packed pair arithmetic.  Clamped at -125 as above.
__device__ __forceinline__ float2 exp2_poly2_x2(float2 x) {
    x = make_float2(fmaxf(x.x, -125.f), fmaxf(x.y, -125.f));
    const float2 magic = make_float2(12582912.f, 12582912.f);
    const float2 j = fadd2(x, magic);                       // n in the low mantissa bits
    const float2 f = fsub2(x, fsub2(j, magic));             // exact: x - n
    float2 p = ffma2(make_float2(0.2384272813796997f, 0.2384272813796997f), f,
                     make_float2(0.7034459114074707f, 0.7034459114074707f));
    p = ffma2(p, f, make_float2(1.0004431009292603f, 1.0004431009292603f));
    return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(j.x) << 23)),
                       __int_as_float(__float_as_int(p.y) + (__float_as_int(j.y) << 23)));
}

// Two floats -> packed bf16x2, round to nearest even; `lo` lands in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two fp32 -> e4m3 (round to nearest even, saturating to +-448): lo in bits 0-7, hi in bits 8-15.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }
__device__ __forceinline__ int warp_id() { return __shfl_sync(0xffffffffu, threadIdx.x >> 5, 0); }

}  // namespace wan
