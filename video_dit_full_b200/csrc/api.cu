// C-ABI layer: argument validation, TMA tensor maps, launches, status word.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <mutex>
#include <set>
#include <utility>

#include "wan_attn.h"
#include "sm100_ptx.cuh"
#include "wan_attn_internal.h"

namespace wan {

__device__ int g_device_status = 0;

int* device_status_word() {
    static std::mutex mu;
    static int* addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* a = nullptr;
        if (cudaGetSymbolAddress(&a, g_device_status) != cudaSuccess) return nullptr;
        addr[dev] = static_cast<int*>(a);
    }
    return addr[dev];
}

namespace {

std::atomic<unsigned long long> g_wait_budget_ns{2000000000ull};

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Tensor map over a bf16 [B, S, H, D] tensor viewed as 4-D (D, H, S, B), box
// (64 of D, 1 head, `box_tokens` tokens, 1 batch) with the 128-byte swizzle.
// Coordinates past S read as zero.
bool make_bshd_map(CUtensorMap* m, const void* base, int B, int S, int H, int D, int box_tokens) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)S * H * D * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)box_tokens, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map over an 8-bit [B*H, S, 128] tensor viewed as 3-D (128, S, B*H), box (128, rows, 1),
// 128-byte swizzle (one 128-byte row per token), tokens past S read as zero.
bool make_bh_s_d8_map(CUtensorMap* m, const void* base, int BH, int S, int rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {128, (cuuint64_t)S, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {128, (cuuint64_t)S * 128};
    const cuuint32_t box[3] = {128, (cuuint32_t)rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map over the fp32 dQ accumulator [B, S, H, 128] as 4-D (128, H, S, B), box
// (128, 1, 128, 1) without swizzle: the backward adds [128 query][128 d] tiles into it.
bool make_dq_acc_map(CUtensorMap* m, void* base, int B, int S, int H) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
    const cuuint64_t strides[3] = {128 * 4, (cuuint64_t)H * 128 * 4, (cuuint64_t)S * H * 128 * 4};
    const cuuint32_t box[4] = {128, 1, 128, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map over an fp32 [B, S, H, 128] accumulator as 4-D (128, H, S, B), box (32, 1, 128, 1)
// with the 128-byte swizzle: the split backward adds [128 key][32 d] sub-tiles of dK, dV into it.
bool make_acc_sw_map(CUtensorMap* m, void* base, int B, int S, int H) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
    const cuuint64_t strides[3] = {128 * 4, (cuuint64_t)H * 128 * 4, (cuuint64_t)S * H * 128 * 4};
    const cuuint32_t box[4] = {32, 1, 128, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map over an 8-bit [rows, K] matrix (K contiguous) as 2-D (K, rows), box (128, box_rows),
// 128-byte swizzle; elements past the edges read as zero.
bool make_rows_u8_map(CUtensorMap* m, const void* base, int rows, int K, int box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)K};
    const cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Shape checks of the FP8 GEMM calls: rows, K >= 1, K % 16 == 0 (16-byte code rows),
// rows * K < 2^40.
int check_fp8_shape(long long rows, long long K) {
    if (rows < 1 || K < 16 || (K & 15) || rows > 0x7fffffffLL || K > 0x7fffffffLL) return WAN_ATTN_ERR_INVALID_ARG;
    if (double(rows) * double(K) >= double(1ull << 40)) return WAN_ATTN_ERR_INVALID_ARG;
    return WAN_ATTN_OK;
}

struct Range {
    uintptr_t lo, hi;
};
Range range_of(const void* p, size_t bytes) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return {a, a + bytes};
}
bool overlaps(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Shape checks common to every call.  Returns a wan_attn_status.
int check_shape(int B, int S, int H, int D) {
    if (B < 1 || S < 1 || H < 1 || D < 1) return WAN_ATTN_ERR_INVALID_ARG;
    if (D != 128) return WAN_ATTN_ERR_UNSUPPORTED;
    if (B > 65535 || H > 65535) return WAN_ATTN_ERR_INVALID_ARG;       // grid y/z limits
    const double n = double(B) * S * H * D;
    if (n >= double(1ull << 40)) return WAN_ATTN_ERR_INVALID_ARG;
    return WAN_ATTN_OK;
}

}  // namespace

int configure_smem(const void* kernel, int bytes) {
    static std::mutex mu;
    static std::set<std::pair<int, const void*>> done;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({dev, kernel})) return 0;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return -1;
    done.insert({dev, kernel});
    return 0;
}

unsigned long long wait_budget_ns() { return g_wait_budget_ns.load(); }

// ---------------------------------------------------------------------------
// bounded-wait self test: one warp waits on a barrier that nobody arrives at
// ---------------------------------------------------------------------------
__global__ void selftest_wait_kernel(unsigned long long budget_ns, int* status) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    const WaitCtl wc{&abort_flag, budget_ns, status};
    (void)wait_warp(b, 0, wc);     // gives up after budget_ns and records the timeout
    __syncthreads();
}

}  // namespace wan

using namespace wan;

namespace {

// Forward of Sq queries against Skv keys (self-attention: Skv = Sq).  The cross-attention call
// with a short key sequence (Skv <= 1024, Sq != Skv: the text embedding) runs the per-tile
// kernel: with a few key blocks per tile, a CTA's prologue and epilogue are much of its time,
// and two CTAs per SM hide each other's.
int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Sq, int Skv, int H,
             int D, void* stream, bool cross) {
    if (!q || !k || !v || !o || !lse) return WAN_ATTN_ERR_INVALID_ARG;
    int st = check_shape(B, Sq, H, D);
    if (st == WAN_ATTN_OK) st = check_shape(B, Skv, H, D);
    if (st != WAN_ATTN_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return WAN_ATTN_ERR_INVALID_ARG;
    const size_t nq = size_t(B) * Sq * H * D, nkv = size_t(B) * Skv * H * D;
    const Range rq = range_of(q, nq * 2), rk = range_of(k, nkv * 2), rv = range_of(v, nkv * 2);
    const Range ro = range_of(o, nq * 2), rl = range_of(lse, size_t(B) * H * Sq * 4);
    for (const Range& in : {rq, rk, rv})
        if (overlaps(ro, in) || overlaps(rl, in)) return WAN_ATTN_ERR_INVALID_ARG;
    if (overlaps(ro, rl)) return WAN_ATTN_ERR_INVALID_ARG;

    const bool per_tile = cross && Sq != Skv && Skv <= 1024;
    const int kv_box = per_tile ? 64 : 128;
    CUtensorMap tq, tk, tv, to;
    if (!make_bshd_map(&tq, q, B, Sq, H, D, 128) || !make_bshd_map(&tk, k, B, Skv, H, D, kv_box) ||
        !make_bshd_map(&tv, v, B, Skv, H, D, kv_box) || !make_bshd_map(&to, o, B, Sq, H, D, 128))
        return WAN_ATTN_ERR_CUDA;
    FwdParams p{};
    p.o = o;
    p.lse = lse;
    p.B = B;
    p.S = Sq;
    p.Skv = Skv;
    p.H = H;
    p.scale_log2 = static_cast<float>((1.0 / std::sqrt(double(D))) * 1.4426950408889634);
    p.wait_budget_ns = wait_budget_ns();
    p.status = device_status_word();
    if (!p.status) return WAN_ATTN_ERR_CUDA;
    if (per_tile) {
        p.nqb = (Sq + 63) / 64;
        p.nkb = (Skv + 63) / 64;
        p.nctas = (Sq + 127) / 128;
        return launch_fwd_tiles(tq, tk, tv, to, p, static_cast<cudaStream_t>(stream)) == 0 ? WAN_ATTN_OK
                                                                                           : WAN_ATTN_ERR_CUDA;
    }
    return launch_fwd(tq, tk, tv, to, p, static_cast<cudaStream_t>(stream)) == 0 ? WAN_ATTN_OK : WAN_ATTN_ERR_CUDA;
}

// Block-sparse forward: per 128-row Q tile (2 query blocks of 64) the list of attended key
// blocks, int32 [B, H, ntiles, nkb], then the lists' lengths [B, H, ntiles].
size_t sparse_ws_size(int B, int Sq, int Skv, int H, int D) {
    if (check_shape(B, Sq, H, D) != WAN_ATTN_OK || check_shape(B, Skv, H, D) != WAN_ATTN_OK) return 0;
    const size_t ntiles = (size_t(Sq) + 127) / 128, nkb = (size_t(Skv) + 63) / 64;
    return align256(size_t(B) * H * ntiles * nkb * 4) + align256(size_t(B) * H * ntiles * 4);
}

int fwd_block_sparse_impl(const void* q, const void* k, const void* v, void* o, float* lse, const uint8_t* mask,
                          int B, int Sq, int Skv, int H, int D, void* workspace, size_t workspace_bytes,
                          void* stream) {
    if (!q || !k || !v || !o || !lse || !mask) return WAN_ATTN_ERR_INVALID_ARG;
    int st = check_shape(B, Sq, H, D);
    if (st == WAN_ATTN_OK) st = check_shape(B, Skv, H, D);
    if (st != WAN_ATTN_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return WAN_ATTN_ERR_INVALID_ARG;
    const size_t need = sparse_ws_size(B, Sq, Skv, H, D);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return WAN_ATTN_ERR_WORKSPACE;
    const int nqb = (Sq + 63) / 64, nkb = (Skv + 63) / 64, ntiles = (Sq + 127) / 128;
    const size_t nq = size_t(B) * Sq * H * D, nkv = size_t(B) * Skv * H * D;
    const Range ins[] = {range_of(q, nq * 2), range_of(k, nkv * 2), range_of(v, nkv * 2),
                         range_of(mask, size_t(B) * H * nqb * nkb)};
    const Range outs[] = {range_of(o, nq * 2), range_of(lse, size_t(B) * H * Sq * 4), range_of(workspace, need)};
    for (size_t a = 0; a < 3; ++a) {
        for (const Range& in : ins)
            if (overlaps(outs[a], in)) return WAN_ATTN_ERR_INVALID_ARG;
        for (size_t c = a + 1; c < 3; ++c)
            if (overlaps(outs[a], outs[c])) return WAN_ATTN_ERR_INVALID_ARG;
    }
    CUtensorMap tq, tk, tv, to;
    if (!make_bshd_map(&tq, q, B, Sq, H, D, 128) || !make_bshd_map(&tk, k, B, Skv, H, D, 64) ||
        !make_bshd_map(&tv, v, B, Skv, H, D, 64) || !make_bshd_map(&to, o, B, Sq, H, D, 128))
        return WAN_ATTN_ERR_CUDA;
    FwdParams p{};
    p.o = o;
    p.lse = lse;
    p.B = B;
    p.S = Sq;
    p.Skv = Skv;
    p.H = H;
    p.mask = mask;
    p.kv_list = static_cast<const int*>(workspace);
    p.kv_count = reinterpret_cast<const int*>(static_cast<char*>(workspace) +
                                              align256(size_t(B) * H * ntiles * nkb * 4));
    p.nqb = nqb;
    p.nkb = nkb;
    p.nctas = ntiles;
    p.scale_log2 = static_cast<float>((1.0 / std::sqrt(double(D))) * 1.4426950408889634);
    p.wait_budget_ns = wait_budget_ns();
    p.status = device_status_word();
    if (!p.status) return WAN_ATTN_ERR_CUDA;
    return launch_fwd_tiles(tq, tk, tv, to, p, static_cast<cudaStream_t>(stream)) == 0 ? WAN_ATTN_OK
                                                                                       : WAN_ATTN_ERR_CUDA;
}

// Backward workspace: fp32 dQ accumulator [B, Sq, H, D], fp32 D_i [B, H, Sq] and, for the
// cross-attention call, fp32 dK and dV accumulators [B, Skv, H, D]; each part 256-byte aligned.
size_t bwd_ws_size(int B, int Sq, int Skv, int H, int D, bool cross) {
    if (check_shape(B, Sq, H, D) != WAN_ATTN_OK || check_shape(B, Skv, H, D) != WAN_ATTN_OK) return 0;
    const size_t nq = size_t(B) * Sq * H * D, nkv = size_t(B) * Skv * H * D;
    size_t bytes = align256(nq * 4) + align256(size_t(B) * H * Sq * 4);
    if (cross) bytes += 2 * align256(nkv * 4);
    return bytes;
}

int bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
             void* dq, void* dk, void* dv, int B, int Sq, int Skv, int H, int D, void* workspace,
             size_t workspace_bytes, void* stream, bool cross) {
    if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return WAN_ATTN_ERR_INVALID_ARG;
    int st = check_shape(B, Sq, H, D);
    if (st == WAN_ATTN_OK) st = check_shape(B, Skv, H, D);
    if (st != WAN_ATTN_OK) return st;
    for (const void* ptr : {q, k, v, o, dO, static_cast<const void*>(lse), static_cast<const void*>(dq),
                            static_cast<const void*>(dk), static_cast<const void*>(dv)})
        if (!aligned16(ptr)) return WAN_ATTN_ERR_INVALID_ARG;
    const size_t need = bwd_ws_size(B, Sq, Skv, H, D, cross);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return WAN_ATTN_ERR_WORKSPACE;
    const size_t nq = size_t(B) * Sq * H * D, nkv = size_t(B) * Skv * H * D;
    const Range ins[] = {range_of(q, nq * 2), range_of(k, nkv * 2), range_of(v, nkv * 2), range_of(o, nq * 2),
                         range_of(dO, nq * 2), range_of(lse, size_t(B) * H * Sq * 4)};
    const Range outs[] = {range_of(dq, nq * 2), range_of(dk, nkv * 2), range_of(dv, nkv * 2),
                          range_of(workspace, need)};
    for (size_t a = 0; a < 4; ++a) {
        for (const Range& in : ins)
            if (overlaps(outs[a], in)) return WAN_ATTN_ERR_INVALID_ARG;
        for (size_t c = a + 1; c < 4; ++c)
            if (overlaps(outs[a], outs[c])) return WAN_ATTN_ERR_INVALID_ARG;
    }

    char* ws = static_cast<char*>(workspace);
    const size_t off_delta = align256(nq * 4);
    const size_t off_dk = off_delta + align256(size_t(B) * H * Sq * 4);
    const size_t off_dv = off_dk + align256(nkv * 4);
    BwdParams p;
    p.lse = lse;
    p.dq_acc = reinterpret_cast<float*>(ws);
    p.delta = reinterpret_cast<float*>(ws + off_delta);
    p.dk_acc = cross ? reinterpret_cast<float*>(ws + off_dk) : nullptr;
    p.dv_acc = cross ? reinterpret_cast<float*>(ws + off_dv) : nullptr;
    CUtensorMap tq, tk, tv, tdo, tdq, tdk, tdv;
    if (!make_bshd_map(&tq, q, B, Sq, H, D, 128) || !make_bshd_map(&tk, k, B, Skv, H, D, 128) ||
        !make_bshd_map(&tv, v, B, Skv, H, D, 128) || !make_bshd_map(&tdo, dO, B, Sq, H, D, 128) ||
        !make_dq_acc_map(&tdq, workspace, B, Sq, H))
        return WAN_ATTN_ERR_CUDA;
    if (cross) {
        if (!make_acc_sw_map(&tdk, p.dk_acc, B, Skv, H) || !make_acc_sw_map(&tdv, p.dv_acc, B, Skv, H))
            return WAN_ATTN_ERR_CUDA;
    } else {
        tdk = tdq;    // never read: self-attention keeps one CTA per key tile (nsplit = 1)
        tdv = tdq;
    }
    p.dk = dk;
    p.dv = dv;
    p.B = B;
    p.Sq = Sq;
    p.Skv = Skv;
    p.H = H;
    p.nsplit = 1;
    p.scale = static_cast<float>(1.0 / std::sqrt(double(D)));
    p.scale_log2 = static_cast<float>((1.0 / std::sqrt(double(D))) * 1.4426950408889634);
    p.wait_budget_ns = wait_budget_ns();
    p.status = device_status_word();
    if (!p.status) return WAN_ATTN_ERR_CUDA;
    return launch_bwd(tq, tk, tv, tdo, tdq, tdk, tdv, p, cross, o, dO, dq, static_cast<cudaStream_t>(stream)) == 0
               ? WAN_ATTN_OK
               : WAN_ATTN_ERR_CUDA;
}

}  // namespace

extern "C" {

int wan_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int S, int H, int D,
                 void* stream) {
    return fwd_impl(q, k, v, o, lse, B, S, S, H, D, stream, false);
}

int wan_attn_cross_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Sq, int Skv,
                       int H, int D, void* stream) {
    return fwd_impl(q, k, v, o, lse, B, Sq, Skv, H, D, stream, true);
}

size_t wan_attn_bwd_workspace_size(int B, int S, int H, int D) { return bwd_ws_size(B, S, S, H, D, false); }

size_t wan_attn_fwd_block_sparse_workspace_size(int B, int Sq, int Skv, int H, int D) {
    return sparse_ws_size(B, Sq, Skv, H, D);
}

int wan_attn_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse,
                              const uint8_t* block_mask, int B, int Sq, int Skv, int H, int D, void* workspace,
                              size_t workspace_bytes, void* stream) {
    return fwd_block_sparse_impl(q, k, v, o, lse, block_mask, B, Sq, Skv, H, D, workspace, workspace_bytes, stream);
}

int wan_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                 void* dq, void* dk, void* dv, int B, int S, int H, int D, void* workspace,
                 size_t workspace_bytes, void* stream) {
    return bwd_impl(q, k, v, o, dO, lse, dq, dk, dv, B, S, S, H, D, workspace, workspace_bytes, stream, false);
}

size_t wan_attn_cross_bwd_workspace_size(int B, int Sq, int Skv, int H, int D) {
    return bwd_ws_size(B, Sq, Skv, H, D, true);
}

int wan_attn_cross_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                       const float* lse, void* dq, void* dk, void* dv, int B, int Sq, int Skv, int H, int D,
                       void* workspace, size_t workspace_bytes, void* stream) {
    return bwd_impl(q, k, v, o, dO, lse, dq, dk, dv, B, Sq, Skv, H, D, workspace, workspace_bytes, stream, true);
}

size_t wan_attn_fwd_q8_workspace_size(int B, int S, int H, int D) {
    if (check_shape(B, S, H, D) != WAN_ATTN_OK) return 0;
    const size_t n = size_t(B) * S * H * D;
    const size_t nblk = (size_t(S) + 63) / 64;
    return 3 * align256(n) + 3 * align256(size_t(B) * H * nblk * 4);
}

int wan_attn_fwd_q8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int S, int H, int D,
                    void* workspace, size_t workspace_bytes, void* stream) {
    if (!q || !k || !v || !o || !lse) return WAN_ATTN_ERR_INVALID_ARG;
    const int st = check_shape(B, S, H, D);
    if (st != WAN_ATTN_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return WAN_ATTN_ERR_INVALID_ARG;
    const size_t need = wan_attn_fwd_q8_workspace_size(B, S, H, D);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return WAN_ATTN_ERR_WORKSPACE;
    const size_t n = size_t(B) * S * H * D;
    const Range ins[] = {range_of(q, n * 2), range_of(k, n * 2), range_of(v, n * 2)};
    const Range outs[] = {range_of(o, n * 2), range_of(lse, size_t(B) * H * S * 4), range_of(workspace, need)};
    for (size_t a = 0; a < 3; ++a) {
        for (const Range& in : ins)
            if (overlaps(outs[a], in)) return WAN_ATTN_ERR_INVALID_ARG;
        for (size_t c = a + 1; c < 3; ++c)
            if (overlaps(outs[a], outs[c])) return WAN_ATTN_ERR_INVALID_ARG;
    }
    const int nblk = (S + 63) / 64;
    char* ws = static_cast<char*>(workspace);
    const size_t code_bytes = align256(n), scale_bytes = align256(size_t(B) * H * nblk * 4);
    Q8QuantParams qp;
    qp.q = static_cast<const __nv_bfloat16*>(q);
    qp.k = static_cast<const __nv_bfloat16*>(k);
    qp.v = static_cast<const __nv_bfloat16*>(v);
    qp.q8 = reinterpret_cast<int8_t*>(ws);
    qp.k8 = reinterpret_cast<int8_t*>(ws + code_bytes);
    qp.v8 = reinterpret_cast<uint8_t*>(ws + 2 * code_bytes);
    qp.sq = reinterpret_cast<float*>(ws + 3 * code_bytes);
    qp.sk = reinterpret_cast<float*>(ws + 3 * code_bytes + scale_bytes);
    qp.sv = reinterpret_cast<float*>(ws + 3 * code_bytes + 2 * scale_bytes);
    qp.B = B;
    qp.S = S;
    qp.H = H;
    qp.nblk = nblk;
    CUtensorMap tq, tk, tv, to;
    if (!make_bh_s_d8_map(&tq, qp.q8, B * H, S, 128) || !make_bh_s_d8_map(&tk, qp.k8, B * H, S, 64) ||
        !make_bh_s_d8_map(&tv, qp.v8, B * H, S, 64) || !make_bshd_map(&to, o, B, S, H, D, 128))
        return WAN_ATTN_ERR_CUDA;
    Q8AttnParams p;
    p.o = o;
    p.lse = lse;
    p.sq = qp.sq;
    p.sk = qp.sk;
    p.sv = qp.sv;
    p.B = B;
    p.S = S;
    p.H = H;
    p.nblk = nblk;
    p.scale_log2 = static_cast<float>((1.0 / std::sqrt(double(D))) * 1.4426950408889634);
    p.wait_budget_ns = wait_budget_ns();
    p.status = device_status_word();
    if (!p.status) return WAN_ATTN_ERR_CUDA;
    return launch_q8(qp, tq, tk, tv, to, p, static_cast<cudaStream_t>(stream)) == 0 ? WAN_ATTN_OK
                                                                                    : WAN_ATTN_ERR_CUDA;
}

int wan_attn_cp_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, void* o_out, int B,
                      int S, int H, int D, int first, void* stream) {
    if (!o_acc || !lse_acc || !o_part || !lse_part) return WAN_ATTN_ERR_INVALID_ARG;
    const int st = check_shape(B, S, H, D);
    if (st != WAN_ATTN_OK) return st;
    for (const void* ptr : {static_cast<const void*>(o_acc), static_cast<const void*>(lse_acc), o_part,
                            static_cast<const void*>(lse_part), static_cast<const void*>(o_out)})
        if (ptr && !aligned16(ptr)) return WAN_ATTN_ERR_INVALID_ARG;
    const size_t n = size_t(B) * S * H * D, nl = size_t(B) * H * S;
    const Range ra = range_of(o_acc, n * 4), rl = range_of(lse_acc, nl * 4);
    const Range ins[] = {range_of(o_part, n * 2), range_of(lse_part, nl * 4)};
    for (const Range& in : ins)
        if (overlaps(ra, in) || overlaps(rl, in)) return WAN_ATTN_ERR_INVALID_ARG;
    if (overlaps(ra, rl)) return WAN_ATTN_ERR_INVALID_ARG;
    if (o_out) {
        const Range ro = range_of(o_out, n * 2);
        if (overlaps(ro, ra) || overlaps(ro, rl) || overlaps(ro, ins[0]) || overlaps(ro, ins[1]))
            return WAN_ATTN_ERR_INVALID_ARG;
    }
    return launch_cp_merge(o_acc, lse_acc, o_part, lse_part, o_out, B, S, H, first ? 1 : 0,
                           static_cast<cudaStream_t>(stream)) == 0
               ? WAN_ATTN_OK
               : WAN_ATTN_ERR_CUDA;
}

int wan_attn_cp_accumulate(float* acc, const void* part, void* out, size_t n, int first, void* stream) {
    if (!acc || !part || n == 0 || (n & 7u)) return WAN_ATTN_ERR_INVALID_ARG;
    if (!aligned16(acc) || !aligned16(part) || (out && !aligned16(out))) return WAN_ATTN_ERR_INVALID_ARG;
    const Range ra = range_of(acc, n * 4), rp = range_of(part, n * 2);
    if (overlaps(ra, rp)) return WAN_ATTN_ERR_INVALID_ARG;
    if (out) {
        const Range ro = range_of(out, n * 2);
        if (overlaps(ro, ra) || overlaps(ro, rp)) return WAN_ATTN_ERR_INVALID_ARG;
    }
    return launch_cp_accumulate(acc, part, out, static_cast<long long>(n / 8), first ? 1 : 0,
                                static_cast<cudaStream_t>(stream)) == 0
               ? WAN_ATTN_OK
               : WAN_ATTN_ERR_CUDA;
}

int wan_attn_cp_layout(void* dst, const void* src, int B, int S_loc, int G, int Hg, int D, int which,
                       void* stream) {
    if (!dst || !src || G < 1 || Hg < 1 || which < WAN_ATTN_CP_SEQ_TO_SEND || which > WAN_ATTN_CP_RECV_TO_SEQ)
        return WAN_ATTN_ERR_INVALID_ARG;
    if (static_cast<long long>(G) * Hg > 65535) return WAN_ATTN_ERR_INVALID_ARG;
    const int st = check_shape(B, S_loc, G * Hg, D);
    if (st != WAN_ATTN_OK) return st;
    if (double(B) * S_loc * G * Hg * D >= double(1ull << 40) / G) return WAN_ATTN_ERR_INVALID_ARG;
    if (!aligned16(dst) || !aligned16(src)) return WAN_ATTN_ERR_INVALID_ARG;
    const size_t bytes = size_t(B) * S_loc * G * Hg * D * 2;
    if (overlaps(range_of(dst, bytes), range_of(src, bytes))) return WAN_ATTN_ERR_INVALID_ARG;
    return launch_cp_layout(dst, src, B, S_loc, G, Hg * D * 2 / 16, which, static_cast<cudaStream_t>(stream)) == 0
               ? WAN_ATTN_OK
               : WAN_ATTN_ERR_CUDA;
}

int wan_fp8_quantize_rows(const void* x, void* codes, float* scales, int M, int K, void* stream) {
    if (!x || !codes || !scales) return WAN_ATTN_ERR_INVALID_ARG;
    const int st = check_fp8_shape(M, K);
    if (st != WAN_ATTN_OK) return st;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return WAN_ATTN_ERR_INVALID_ARG;
    const size_t n = size_t(M) * K;
    const Range rx = range_of(x, n * 2), rc = range_of(codes, n), rs = range_of(scales, size_t(M) * 4);
    if (overlaps(rx, rc) || overlaps(rx, rs) || overlaps(rc, rs)) return WAN_ATTN_ERR_INVALID_ARG;
    return launch_fp8_quant_rows(x, codes, scales, M, K, static_cast<cudaStream_t>(stream)) == 0 ? WAN_ATTN_OK
                                                                                               : WAN_ATTN_ERR_CUDA;
}

int wan_fp8_quantize_tensor(const void* w, void* codes, float* scale2, int N, int K, void* stream) {
    if (!w || !codes || !scale2) return WAN_ATTN_ERR_INVALID_ARG;
    const int st = check_fp8_shape(N, K);
    if (st != WAN_ATTN_OK) return st;
    if (!aligned16(w) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scale2) & 7u))
        return WAN_ATTN_ERR_INVALID_ARG;
    const size_t n = size_t(N) * K;
    const Range rw = range_of(w, n * 2), rc = range_of(codes, n), rs = range_of(scale2, 8);
    if (overlaps(rw, rc) || overlaps(rw, rs) || overlaps(rc, rs)) return WAN_ATTN_ERR_INVALID_ARG;
    return launch_fp8_quant_tensor(w, codes, scale2, static_cast<long long>(n), static_cast<cudaStream_t>(stream)) == 0
               ? WAN_ATTN_OK
               : WAN_ATTN_ERR_CUDA;
}

int wan_fp8_gemm(const void* a_codes, const float* a_scales, const void* b_codes, const float* b_scale, void* y,
                 int M, int N, int K, void* stream) {
    if (!a_codes || !a_scales || !b_codes || !b_scale || !y) return WAN_ATTN_ERR_INVALID_ARG;
    int st = check_fp8_shape(M, K);
    if (st == WAN_ATTN_OK) st = check_fp8_shape(N, K);
    if (st != WAN_ATTN_OK) return st;
    if ((N & 7) || double(M) * N >= double(1ull << 40)) return WAN_ATTN_ERR_INVALID_ARG;
    if (!aligned16(a_codes) || !aligned16(b_codes) || !aligned16(y) || (reinterpret_cast<uintptr_t>(a_scales) & 3u) ||
        (reinterpret_cast<uintptr_t>(b_scale) & 3u))
        return WAN_ATTN_ERR_INVALID_ARG;
    const Range ry = range_of(y, size_t(M) * N * 2);
    const Range ins[] = {range_of(a_codes, size_t(M) * K), range_of(a_scales, size_t(M) * 4),
                         range_of(b_codes, size_t(N) * K), range_of(b_scale, 4)};
    for (const Range& in : ins)
        if (overlaps(ry, in)) return WAN_ATTN_ERR_INVALID_ARG;
    CUtensorMap ta, tb, tb_half;
    if (!make_rows_u8_map(&ta, a_codes, M, K, 128) || !make_rows_u8_map(&tb, b_codes, N, K, 256) ||
        !make_rows_u8_map(&tb_half, b_codes, N, K, 128))
        return WAN_ATTN_ERR_CUDA;
    Fp8GemmParams p;
    p.a_scales = a_scales;
    p.b_scale = b_scale;
    p.y = y;
    p.M = M;
    p.N = N;
    p.K = K;
    p.wait_budget_ns = wait_budget_ns();
    p.status = device_status_word();
    if (!p.status) return WAN_ATTN_ERR_CUDA;
    return launch_fp8_gemm(ta, tb, tb_half, p, static_cast<cudaStream_t>(stream)) == 0 ? WAN_ATTN_OK
                                                                                     : WAN_ATTN_ERR_CUDA;
}

int wan_attn_sync_status(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return WAN_ATTN_ERR_CUDA;
    int h = 0;
    if (cudaMemcpyFromSymbol(&h, g_device_status, sizeof(int)) != cudaSuccess) return WAN_ATTN_ERR_CUDA;
    if (h != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return WAN_ATTN_ERR_CUDA;
    }
    return h;
}

const char* wan_attn_status_string(int status) {
    switch (status) {
        case WAN_ATTN_OK: return "ok";
        case WAN_ATTN_ERR_INVALID_ARG: return "invalid argument";
        case WAN_ATTN_ERR_UNSUPPORTED: return "unsupported (head dim must be 128)";
        case WAN_ATTN_ERR_CUDA: return "CUDA error";
        case WAN_ATTN_ERR_TIMEOUT: return "a kernel wait ran out of time";
        case WAN_ATTN_ERR_WORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

uint64_t wan_attn_set_wait_budget_ns(uint64_t ns) {
    if (ns < 1000) ns = 1000;
    return g_wait_budget_ns.exchange(ns);
}

int wan_attn_selftest_wait_timeout(uint64_t budget_ns, void* stream) {
    if (budget_ns < 1000) budget_ns = 1000;
    int* status = device_status_word();
    if (!status) return WAN_ATTN_ERR_CUDA;
    selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(budget_ns, status);
    return cudaGetLastError() == cudaSuccess ? WAN_ATTN_OK : WAN_ATTN_ERR_CUDA;
}

}  // extern "C"
