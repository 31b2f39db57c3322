/*
 * wan_attn.h - C ABI of the B200 (sm_100a) full self-attention library for
 * Wan-style video diffusion transformers.
 *
 * The operation.  Inside every DiT block of Wan, all tokens of the patchified
 * video latent attend to all other tokens, bidirectionally:
 *     O = softmax(Q K^T / sqrt(D)) V,
 * non-causal and neither windowed nor masked.  Sources: "Wan 2.1: VBench
 * 86.22% ..." (paper-podcast summary of the Wan report), section
 * "干预与形式化" (the DiT's full spatio-temporal self-attention) and section
 * "先看现象" (cost model C = L(alpha*b*s*h^2 + beta*b*s^2*h), non-causal
 * attention with beta = 4 forward and 8 backward; the token count
 * (1+T/4)(H/16)(W/16) of the VAE latent after the (1,2,2) patchify);
 * "Wan: Open and Advanced Large-Scale Video Generative Models", section 5
 * (attention is what grows with sequence length in training).
 *
 * Conventions shared by every call:
 *   - Q, K, V, O (and dO, dQ, dK, dV) are bf16 tensors laid out [B, S, H, D],
 *     contiguous, D fastest.  D must be 128.
 *   - lse is fp32 [B, H, S]: lse[b,h,i] = ln sum_j exp(q_i . k_j / sqrt(D)).
 *   - The softmax scale is fixed at 1/sqrt(D).  No mask, no dropout, no bias.
 *   - Every pointer is a device pointer owned by the caller, 16-byte aligned.
 *     The library allocates no memory.  Outputs may not overlap inputs.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     validate their arguments on the host, enqueue their kernels and return;
 *     they do not synchronise.  On a validation failure nothing is enqueued.
 *   - Kernels never spin without bound: every wait inside a kernel has a time
 *     budget; when one runs out the kernel records WAN_ATTN_ERR_TIMEOUT in a
 *     device status word and exits.  wan_attn_sync_status() reports it.
 *     While the status word holds an error, a wait that has lasted 1 ms
 *     gives up too (healthy waits are far shorter), so that the CTAs of a
 *     call that timed out do not each spend a whole budget.
 *   - The library looks up the device addresses of its own static device
 *     variables (the status word; the no-alloc backward's array) once per
 *     device and keeps them for the life of the process.  Do not keep using
 *     it on a device after cudaDeviceReset.
 */
#ifndef WAN_ATTN_H
#define WAN_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define WAN_ATTN_API __attribute__((visibility("default")))
#else
#define WAN_ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    WAN_ATTN_OK = 0,
    WAN_ATTN_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment, overlap */
    WAN_ATTN_ERR_UNSUPPORTED = 2,   /* D != 128 */
    WAN_ATTN_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed (launch, tensor map) */
    WAN_ATTN_ERR_TIMEOUT = 4,       /* a kernel's bounded wait ran out (reported by sync_status) */
    WAN_ATTN_ERR_WORKSPACE = 5      /* workspace pointer null or smaller than required */
} wan_attn_status;

/*
 * Forward, bf16.
 *   q, k, v : in,  bf16 [B, S, H, D]
 *   o       : out, bf16 [B, S, H, D], rounded to nearest even from fp32
 *   lse     : out, fp32 [B, H, S], natural-log log-sum-exp of the scaled
 *             scores of each query row (the backward's input); not NULL.
 *   B, S, H : >= 1, with B*S*H*D < 2^40;  D : must be 128.
 * Accumulation is fp32 (scores, running max and sum, and O); P = 2^(s - m)
 * is rounded to bf16 for P V.  Of every 16 exponentials 14 come from the
 * hardware exp2 and 2 from a degree-3 polynomial (relative error 7.5e-5).
 * Returns WAN_ATTN_OK once the kernel is enqueued.
 */
WAN_ATTN_API int wan_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int S, int H, int D, void* stream);

/*
 * Bytes of device workspace wan_attn_bwd needs for these sizes: an fp32 dQ
 * accumulator [B, S, H, D] followed by fp32 D_i = rowsum(dO * O) [B, H, S],
 * each starting on a 256-byte boundary.  Returns 0 if the sizes are invalid.
 */
WAN_ATTN_API size_t wan_attn_bwd_workspace_size(int B, int S, int H, int D);

/*
 * Backward, bf16: gradients of sum(O * dO) for O = attention(Q, K, V).
 *   q, k, v : in,  bf16 [B, S, H, D] (the forward's inputs)
 *   o       : in,  bf16 [B, S, H, D] (the forward's output)
 *   dO      : in,  bf16 [B, S, H, D]
 *   lse     : in,  fp32 [B, H, S] written by wan_attn_fwd for the same inputs
 *   dq, dk, dv : out, bf16 [B, S, H, D], rounded to nearest even
 *   workspace, workspace_bytes : caller-owned device memory, 256-byte aligned,
 *             at least wan_attn_bwd_workspace_size(B, S, H, D) bytes
 *             (else WAN_ATTN_ERR_WORKSPACE).  Its contents on entry are
 *             ignored; it must not overlap any other argument.
 * The softmax matrix is recomputed from lse, never stored: P = exp(S/sqrt(D)
 * - lse), dS = P * (dP - D), dV = P^T dO, dK = dS^T Q / sqrt(D), dQ = dS K /
 * sqrt(D) (the non-causal backward of the cost model's beta = 8 term).
 * dQ is accumulated in fp32 in the workspace across key tiles (asynchronous
 * bulk reduce-adds of each tile's partial, in no fixed order), so its low bits
 * may differ between runs; dK and dV are deterministic.
 */
WAN_ATTN_API int wan_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                              const float* lse, void* dq, void* dk, void* dv, int B, int S, int H, int D,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * Cross-attention forward, bf16: the DiT block's attention from the video
 * tokens to the text condition ("Wan 2.1 ..." paper-podcast summary, section
 * "干预与形式化": c_txt is umT5's 512-token text embedding, and the DiT
 * backbone injects umT5 by cross-attention).  Same definition as wan_attn_fwd
 * with the key index running over the Skv key/value tokens:
 *     O = softmax(Q K^T / sqrt(D)) V,  Q [Sq x D] per (b, h), K, V [Skv x D].
 *   q       : in,  bf16 [B, Sq, H, D]
 *   k, v    : in,  bf16 [B, Skv, H, D] (already projected to the attention heads)
 *   o       : out, bf16 [B, Sq, H, D]
 *   lse     : out, fp32 [B, H, Sq], natural log; not NULL
 *   B, Sq, Skv, H >= 1 (each of B*Sq*H*D and B*Skv*H*D < 2^40); D must be 128.
 * No mask: the Skv keys are all attended to (a caller whose text is padded
 * passes the padded embedding, as the 512-token condition is).  Other
 * conventions, precision and errors as wan_attn_fwd; wan_attn_cross_fwd with
 * Skv = Sq and the same pointers computes what wan_attn_fwd does, bit for bit.
 * With Sq != Skv <= 1024 the call runs one CTA per 128-query tile, two per SM,
 * in 128-key steps with every exponential from the hardware exp2, so its
 * rounding differs slightly from wan_attn_fwd's.
 */
WAN_ATTN_API int wan_attn_cross_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                                    int Sq, int Skv, int H, int D, void* stream);

/*
 * Bytes of device workspace wan_attn_cross_bwd needs: fp32 dQ accumulator
 * [B, Sq, H, D], fp32 D_i [B, H, Sq], fp32 dK and dV accumulators
 * [B, Skv, H, D], each starting on a 256-byte boundary.  0 if the sizes are
 * invalid.
 */
WAN_ATTN_API size_t wan_attn_cross_bwd_workspace_size(int B, int Sq, int Skv, int H, int D);

/*
 * Cross-attention backward, bf16: gradients of sum(O * dO) for
 * O = wan_attn_cross_fwd(Q, K, V), with the formulas of wan_attn_bwd.
 *   q, o, dO : in,  bf16 [B, Sq, H, D];  k, v : in, bf16 [B, Skv, H, D]
 *   lse      : in,  fp32 [B, H, Sq] from wan_attn_cross_fwd on the same inputs
 *   dq       : out, bf16 [B, Sq, H, D];  dk, dv : out, bf16 [B, Skv, H, D]
 *   workspace, workspace_bytes : caller-owned device memory, 256-byte aligned,
 *             at least wan_attn_cross_bwd_workspace_size bytes (else
 *             WAN_ATTN_ERR_WORKSPACE); contents on entry ignored.
 * With few key tiles (Skv = 512 gives 4 per head) the call spreads each key
 * tile's queries over several CTAs that add their dK, dV parts in fp32 in the
 * workspace; dK and dV (like dQ) may then differ in their low bits between
 * runs.  Other conventions and errors as wan_attn_bwd.
 */
WAN_ATTN_API int wan_attn_cross_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                    const float* lse, void* dq, void* dk, void* dv, int B, int Sq, int Skv,
                                    int H, int D, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Block-sparse forward with a given 64 x 64 block mask: the block-sparse
 * attention of the FastWan / VSA article on the first page ("一夜颠覆Sora神话，
 * H200单卡5秒出片…": each 64-token query block keeps a subset of the 64-token
 * key blocks, 87.5 % sparsity in its runs; FlexAttention compared on the same
 * 64 x 64 block-sparse mask).  The mask is an input (the learned coarse stage
 * that chooses blocks is not part of this library).  Block i of a sequence
 * holds tokens [64 i, 64 i + 64), the last block possibly short.
 *   q : bf16 [B, Sq, H, D];  k, v : bf16 [B, Skv, H, D];  D must be 128
 *   block_mask : uint8 [B, H, ceil(Sq/64), ceil(Skv/64)], non-zero = query block
 *                i attends key block j (no alignment needed)
 *   o : out bf16 [B, Sq, H, D];  lse : out fp32 [B, H, Sq]
 *   A row whose query block attends no key block gets o = 0 and lse = -inf.
 *   workspace, workspace_bytes : caller-owned device memory, 256-byte aligned,
 *     at least wan_attn_fwd_block_sparse_workspace_size bytes: the per-tile
 *     lists of attended key blocks (int32 [B, H, ceil(Sq/128), ceil(Skv/64)])
 *     and their lengths, built on the device by this call.
 * Work: a CTA covers one 128-row Q tile (2 query blocks) and steps through
 * the union of the key blocks its 2 query blocks attend, two listed blocks
 * (128 keys) per step; each row keeps only its own query block's blocks, and
 * a query block that skips one of a step's blocks gets P = 0 for its 64 keys.
 * Every exponential comes from the hardware exp2.  Other conventions as
 * wan_attn_fwd.
 */
WAN_ATTN_API size_t wan_attn_fwd_block_sparse_workspace_size(int B, int Sq, int Skv, int H, int D);
WAN_ATTN_API int wan_attn_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse,
                                           const uint8_t* block_mask, int B, int Sq, int Skv, int H, int D,
                                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Context parallelism: the building blocks of the two schemes the pages name for
 * sequences too long for one GPU (kwkr.cn Wan explainer, section 3.2: the token
 * sequence is split over GPUs and combined with Ulysses and Ring Attention;
 * "Wan: Open and Advanced Large-Scale Video Generative Models", section 5: the
 * DiT trains with FSDP + 2-D context parallel, converting layouts at module
 * boundaries).  The exchanges themselves (all-to-all, ring send/recv) are NCCL
 * calls made by the caller (video_dit_full_b200.context_parallel).
 *
 * Ring Attention.  A rank holding queries Q_r meets the key blocks K_t, V_t one
 * at a time; wan_attn_cross_fwd gives each block's partial (O_t, lse_t) and
 *     lse' = logaddexp(lse, lse_t),   O' = e^(lse - lse') O + e^(lse_t - lse') O_t
 * folds it into a running fp32 (O, lse): exactly the softmax over every key
 * seen so far.
 *   o_acc    : in/out fp32 [B, S, H, D]   (ignored on input when first != 0)
 *   lse_acc  : in/out fp32 [B, H, S]      (ignored on input when first != 0)
 *   o_part   : in  bf16 [B, S, H, D];  lse_part : in fp32 [B, H, S] (natural log)
 *   o_out    : out bf16 [B, S, H, D] = the updated o_acc rounded to nearest even,
 *              or NULL for none
 *   first    : non-zero = start a new sum (o_acc = o_part, lse_acc = lse_part)
 *   D must be 128.  Pointers 16-byte aligned; outputs overlap nothing.
 */
WAN_ATTN_API int wan_attn_cp_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                                   void* o_out, int B, int S, int H, int D, int first, void* stream);

/*
 * acc = (first ? 0 : acc) + part over n elements (part bf16, acc fp32), and
 * out = bf16(acc) when out is not NULL: the ring backward's sums of dQ parts
 * and of the dK, dV parts that travel with their key block.  n must be a
 * positive multiple of 8; pointers 16-byte aligned; no overlaps.
 */
WAN_ATTN_API int wan_attn_cp_accumulate(float* acc, const void* part, void* out, size_t n, int first,
                                        void* stream);

/*
 * Ulysses.  A rank holds S_loc tokens of all H = G*Hg heads; one all-to-all
 * (equal chunks, chunk g to rank g) gives every rank all G*S_loc tokens of its
 * Hg heads, attention runs locally, and a second all-to-all brings O back.
 * wan_attn_cp_layout moves [Hg x D] bf16 blocks between the orders around
 * those exchanges (B = batch, g = rank / head group, s = token within a shard):
 *   WAN_ATTN_CP_SEQ_TO_SEND   [B, S_loc, G, Hg, D] -> [G, B, S_loc, Hg, D]  (send buffer)
 *   WAN_ATTN_CP_RECV_TO_HEADS [G, B, S_loc, Hg, D] -> [B, G*S_loc, Hg, D]   (attention input)
 *   WAN_ATTN_CP_HEADS_TO_SEND [B, G*S_loc, Hg, D] -> [G, B, S_loc, Hg, D]   (send buffer)
 *   WAN_ATTN_CP_RECV_TO_SEQ   [G, B, S_loc, Hg, D] -> [B, S_loc, G*Hg, D]   (back in sequence shards)
 * dst and src hold B*S_loc*G*Hg*D bf16 each, 16-byte aligned, not overlapping;
 * D must be 128.
 */
#define WAN_ATTN_CP_SEQ_TO_SEND 0
#define WAN_ATTN_CP_RECV_TO_HEADS 1
#define WAN_ATTN_CP_HEADS_TO_SEND 2
#define WAN_ATTN_CP_RECV_TO_SEQ 3
WAN_ATTN_API int wan_attn_cp_layout(void* dst, const void* src, int B, int S_loc, int G, int Hg, int D, int which,
                                    void* stream);

/*
 * FP8 GEMM of the DiT linear layers: the pages' FP8 GEMM (kwkr.cn Wan
 * explainer, section 4.2: the most expensive matrix products run in FP8,
 * weights quantised per tensor and activations per token; Wan 2.1
 * paper-podcast summary, section "干预与形式化": FP8 GEMM, 1.13x).  For
 * activations X [M, K] (tokens x in-features) and a weight W [N, K]
 * (out-features x in-features, the nn.Linear layout):
 *     sx[m] = absmax_k |X[m,k]| / 448,  xq = e4m3(x * fp32(448 / absmax))
 *     sw    = absmax |W| / 448,         wq = e4m3(w * fp32(448 / absmax))
 *     Y[m, n] = bf16(sx[m] * sw * sum_k xq[m,k] * wq[n,k])   (fp32 accumulation)
 * e4m3 is the fn variant (largest finite 448), round to nearest even,
 * saturating; the scale of an all-zero row / tensor is 1.  Codes are bytes,
 * rows of K contiguous codes.  K must be a multiple of 16 (>= 16); every
 * pointer 16-byte aligned unless stated; outputs overlap no input.
 */
/* Per-row (token) quantiser: x bf16 [M, K] -> codes u8 [M, K], scales fp32 [M]. */
WAN_ATTN_API int wan_fp8_quantize_rows(const void* x, void* codes, float* scales, int M, int K, void* stream);

/*
 * Per-tensor quantiser: w bf16 [N, K] -> codes u8 [N, K].  scale2 points to two
 * fp32 in device memory (8-byte aligned): on return scale2[0] = sw and
 * scale2[1] holds absmax |W| (its bits are the kernels' scratch meanwhile).
 */
WAN_ATTN_API int wan_fp8_quantize_tensor(const void* w, void* codes, float* scale2, int N, int K, void* stream);

/*
 * Y = diag(a_scales) (a_codes b_codes^T) (*b_scale):
 *   a_codes u8 [M, K], a_scales fp32 [M] (4-byte aligned), b_codes u8 [N, K],
 *   b_scale: one fp32 in device memory (e.g. scale2 above), y bf16 [M, N].
 *   N must be a multiple of 8; M, N >= 1; M*N < 2^40.
 * Tensor cores: tcgen05.mma kind::f8f6f4, 128 x 256 output tiles per CTA.
 */
WAN_ATTN_API int wan_fp8_gemm(const void* a_codes, const float* a_scales, const void* b_codes,
                              const float* b_scale, void* y, int M, int N, int K, void* stream);

/*
 * Bytes of device workspace wan_attn_fwd_q8 needs: the quantised copies and
 * their scales, each part starting on a 256-byte boundary, in this order:
 *   int8 Q8 [B, H, S, D], int8 K8 [B, H, S, D], e4m3 V8 [B, H, S, D],
 *   fp32 sQ, sK, sV [B, H, ceil(S/64)].
 * Returns 0 if the sizes are invalid.
 */
WAN_ATTN_API size_t wan_attn_fwd_q8_workspace_size(int B, int S, int H, int D);

/*
 * 8-bit forward: the pages' 8-bit FlashAttention ("Wan 2.1 ..." paper-podcast
 * summary, section "干预与形式化": mixed int8/FP8 with FP32 accumulation
 * across blocks; kwkr.cn Wan explainer, section 4.2).  Read as:
 *   - per (b, h, 64-token block): sQ = absmax(Q)/127, sK = absmax(K)/127,
 *     sV = the smallest power of two >= absmax(V)/448, at least 2^-126
 *     (fp32; every scale is 1 for an all-zero block); codes
 *     Q8 = clamp(rint(q * fp32(127 / absmax(Q))), -127, 127) with an fp32
 *     product, K8 likewise, V8 = e4m3(v / sV) (exact: sV is a power of two),
 *     rounding to nearest even, e4m3 saturating;
 *   - scores S = (Q8 . K8) sQ sK / sqrt(D) from int32 tensor-core sums;
 *   - P8 = e4m3(224 * exp(S - m) * sV_block / sV_max), where m is the running
 *     row max (moved only when it rises by more than a factor 2) and sV_max
 *     the head's largest V block scale: each block's V scale rides in P;
 *   - every block's P8 V8 is summed by the tensor core's fp32 accumulator
 *     (fp32 accumulation across blocks); O = that sum * sV_max / 224 / l,
 *     with the row sum l taken over the unquantised exponentials;
 *   - exp is evaluated in fp32, for 3 in 8 of the scores by a degree-2
 *     polynomial with relative error <= 1.73e-3 (below e4m3's half step),
 *     so the LSE carries up to ln(1 + 1.73e-3) beyond the score error.
 *   q, k, v : in,  bf16 [B, S, H, D]
 *   o       : out, bf16 [B, S, H, D]
 *   lse     : out, fp32 [B, H, S], natural log, of the dequantised scores
 *   workspace, workspace_bytes : caller-owned device memory, 256-byte aligned,
 *             at least wan_attn_fwd_q8_workspace_size bytes (else
 *             WAN_ATTN_ERR_WORKSPACE); on return it holds the quantised
 *             tensors and scales in the layout above.
 * Other conventions as wan_attn_fwd.
 */
WAN_ATTN_API int wan_attn_fwd_q8(const void* q, const void* k, const void* v, void* o, float* lse,
                                 int B, int S, int H, int D, void* workspace, size_t workspace_bytes,
                                 void* stream);

/*
 * Size of the library's own backward workspace used by wan_attn_bwd_noalloc:
 * 32 MiB of static device memory in the library's module.  The CUDA runtime
 * loads that module on a device at the latest when the first
 * wan_attn_bwd_noalloc call on that device looks the array up (earlier when
 * lazy module loading is off); from then on the device holds the 32 MiB until
 * the process exits.  It fits B*S*H <= 65027 (token, head) rows, e.g. B=1,
 * S=2048, H=31.
 */
#define WAN_ATTN_NOALLOC_WORKSPACE_BYTES (32u << 20)

/*
 * The backward of wan_attn_bwd without a caller-supplied workspace: no
 * counterpart in the pages; it serves callers that cannot allocate device
 * memory (a plugin whose host application owns all device memory and hands
 * out no allocator, or a server that forbids cudaMalloc after start-up since
 * it can synchronise the device and fragment memory).  Arguments, layouts,
 * results and errors are those of wan_attn_bwd, minus the workspace, which is
 * a fixed WAN_ATTN_NOALLOC_WORKSPACE_BYTES device array inside the library.
 *   - Sizes whose wan_attn_bwd_workspace_size(B, S, H, D) exceeds that array
 *     return WAN_ATTN_ERR_WORKSPACE and enqueue nothing.
 *   - The call allocates and frees nothing itself.  Its first call on a
 *     device looks up the array's device address (cudaGetSymbolAddress) with
 *     that device current, which can load the module and so reserve the
 *     32 MiB (the one implicit reservation); make that first call at
 *     start-up, before any stream capture.  The address is kept per device
 *     for the life of the process: do not keep using the library on a device
 *     after cudaDeviceReset (the module, and with it the array and the
 *     library's status word, may come back at another address).
 *   - Every call on a device shares the one array.  Calls whose kernels
 *     overlap on the GPU (other streams, other host threads) race on it:
 *     order them on one stream or with events.  Each call clears what must
 *     start at zero, so a finished earlier call leaves nothing behind that
 *     matters.
 */
WAN_ATTN_API int wan_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                      const void* dO, const float* lse, void* dq, void* dk, void* dv,
                                      int B, int S, int H, int D, void* stream);

/*
 * Synchronises `stream`, then returns and clears the device status word:
 * WAN_ATTN_OK, WAN_ATTN_ERR_TIMEOUT (a kernel's bounded wait ran out), or
 * WAN_ATTN_ERR_CUDA if the synchronisation itself failed.
 */
WAN_ATTN_API int wan_attn_sync_status(void* stream);

/* Static, human-readable name of a status code. */
WAN_ATTN_API const char* wan_attn_status_string(int status);

/*
 * Time budget, in nanoseconds, of every bounded wait inside the kernels
 * launched after this call on this process (default 2e9 = 2 s; values
 * below 1000 are raised to 1000).  Returns the previous budget.
 */
WAN_ATTN_API uint64_t wan_attn_set_wait_budget_ns(uint64_t ns);

/*
 * Self-test of the bounded-wait path: launches one small CTA that waits on a
 * barrier nobody arrives at, with the given budget, then exits through the
 * same give-up path the attention kernels use.  A following
 * wan_attn_sync_status() returns WAN_ATTN_ERR_TIMEOUT.  No counterpart in the
 * pages: it exists so failure detection can be tested without faulting a GPU.
 */
WAN_ATTN_API int wan_attn_selftest_wait_timeout(uint64_t budget_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* WAN_ATTN_H */
