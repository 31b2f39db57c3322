// Internal declarations shared by the C-ABI layer and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

namespace wan {

struct FwdParams {
    void* o;                    // bf16 [B, S, H, 128]
    float* lse;                 // fp32 [B, H, S], natural log
    int B, S, H;                // S = query tokens
    int Skv;                    // key / value tokens (= S for self-attention)
    // block-sparse forward only: 64 x 64 block mask uint8 [B, H, nqb, nkb], and per 128-row Q
    // tile (2 query blocks) the ascending list of key blocks either attends
    // (kv_list [B, H, nctas, nkb] int32, nctas = the number of Q tiles; each entry the key block
    // with bit 30 set if the tile's first query block attends it, bit 31 if the second does)
    // with its length (kv_count [B, H, nctas])
    const uint8_t* mask;
    const int* kv_list;
    const int* kv_count;
    int nqb, nkb, nctas;
    float scale_log2;           // (1 / sqrt(D)) * log2(e)
    unsigned long long wait_budget_ns;
    int* status;                // device status word (see wan_attn_sync_status)
};

struct BwdParams {
    const float* lse;           // fp32 [B, H, Sq] from the forward (natural log)
    float* delta;               // workspace fp32 [B, H, Sq]: rowsum(dO * O)
    float* dq_acc;              // workspace fp32 [B, Sq, H, 128]: unscaled dS K
    float* dk_acc;              // workspace fp32 [B, Skv, H, 128] (split query ranges only)
    float* dv_acc;              // workspace fp32 [B, Skv, H, 128] (split query ranges only)
    void* dk;                   // bf16 [B, Skv, H, 128]
    void* dv;                   // bf16 [B, Skv, H, 128]
    int B, Sq, Skv, H;
    int nsplit;                 // CTAs sharing one key tile, each over its own range of Q tiles
    float scale;                // 1 / sqrt(D)
    float scale_log2;           // scale * log2(e)
    unsigned long long wait_budget_ns;
    int* status;
};

struct Q8QuantParams {
    const __nv_bfloat16 *q, *k, *v;   // bf16 [B, S, H, 128]
    int8_t *q8, *k8;                  // int8 [B, H, S, 128]
    uint8_t* v8;                      // e4m3 [B, H, S, 128]
    float *sq, *sk, *sv;              // fp32 [B, H, nblk]
    int B, S, H, nblk;
};

struct Q8AttnParams {
    void* o;                          // bf16 [B, S, H, 128]
    float* lse;                       // fp32 [B, H, S]
    const float *sq, *sk, *sv;        // fp32 [B, H, nblk]
    int B, S, H, nblk;
    float scale_log2;
    unsigned long long wait_budget_ns;
    int* status;
};

struct Fp8GemmParams {
    const float* a_scales;            // fp32 [M]: per-row (token) scales of the activation codes
    const float* b_scale;             // fp32 [1]: the weight's per-tensor scale (device memory)
    void* y;                          // bf16 [M, N]
    int M, N, K;
    unsigned long long wait_budget_ns;
    int* status;
};

// Device address of the status word on the current device (nullptr on failure).
int* device_status_word();
unsigned long long wait_budget_ns();

// Sets the dynamic shared-memory limit of a kernel once per device.  0 on success.
int configure_smem(const void* kernel, int bytes);

// `to`: a map over O with the layout and box of tq (the epilogue TMA-stores O through it).
int launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
               const FwdParams& p, cudaStream_t stream);
// Forward with one CTA per 128-row Q tile (p.nctas = the number of Q tiles); tk64 / tv64 are
// K / V maps with 64-token boxes.  Block-sparse (p.kv_list set): builds each tile's
// key-block list in p.kv_list / p.kv_count (device workspace) from p.mask, then runs the
// pair-step kernel over the lists.  p.kv_list null: every key block, no mask, on the per-tile
// kernel with 64-key steps.
int launch_fwd_tiles(const CUtensorMap& tq, const CUtensorMap& tk64, const CUtensorMap& tv64, const CUtensorMap& to,
                     const FwdParams& p, cudaStream_t stream);

// Chooses p.nsplit (1 unless allow_split and the key tiles alone fill too few waves of the
// GPU), then launches the backward's kernels.  tdk / tdv (fp32 accumulators, as tdq) are only
// read when p.nsplit > 1.
int launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
               const CUtensorMap& tdq, const CUtensorMap& tdk, const CUtensorMap& tdv, BwdParams p,
               bool allow_split, const void* o, const void* dout, void* dq, cudaStream_t stream);

// Context-parallel helpers (cp_kernels.cu).  0 on success.
int launch_cp_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, void* o_out, int B,
                    int S, int H, int first, cudaStream_t stream);
int launch_cp_accumulate(float* acc, const void* part, void* out, long long n8, int first, cudaStream_t stream);
int launch_cp_layout(void* dst, const void* src, int B, int S, int G, int blk16, int which, cudaStream_t stream);

// FP8 GEMM of the linear layers (fp8_gemm.cu).  0 on success.
int launch_fp8_quant_rows(const void* x, void* codes, float* scales, int M, int K, cudaStream_t stream);
int launch_fp8_quant_tensor(const void* w, void* codes, float* scale2, long long n, cudaStream_t stream);
// tb: W's map with 256-row boxes (1-CTA kernel); tb_half: 128-row boxes (CTA pairs).
int launch_fp8_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tb_half, const Fp8GemmParams& p,
                    cudaStream_t stream);

// `to`: a map over the bf16 O [B, S, H, D] with 128-token boxes (the epilogue TMA-stores O through it).
int launch_q8(const Q8QuantParams& qp, const CUtensorMap& tq8, const CUtensorMap& tk8, const CUtensorMap& tv8,
              const CUtensorMap& to, const Q8AttnParams& p, cudaStream_t stream);

}  // namespace wan
