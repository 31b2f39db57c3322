// wan_attn_bwd_noalloc: the backward with its workspace in a fixed device array
// owned by this library, for callers that cannot allocate device memory.
//
// Some callers have no way to allocate: a plugin whose host application owns
// every byte of device memory and hands out no allocator, or a serving
// process that forbids cudaMalloc after start-up (it can synchronise the
// device, stall other streams and fragment the heap).  They still own their
// inputs and outputs, but the backward also needs scratch (the fp32 dQ
// accumulator and D_i = rowsum(dO * O)); this entry point takes it from
// g_bwd_scratch below instead of from the caller.
#include <cuda_runtime.h>

#include <mutex>

#include "wan_attn.h"

namespace {

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_bwd_scratch[WAN_ATTN_NOALLOC_WORKSPACE_BYTES];

// Device address of g_bwd_scratch on the current device, looked up once per
// device (in host code the symbol's name is only a stand-in, not an address).
void* scratch_on_current_device() {
    static std::mutex mu;
    static void* addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || !p) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

extern "C" int wan_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                    const float* lse, void* dq, void* dk, void* dv, int B, int S, int H, int D,
                                    void* stream) {
    if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return WAN_ATTN_ERR_INVALID_ARG;
    const size_t need = wan_attn_bwd_workspace_size(B, S, H, D);
    if (need == 0) {   // invalid sizes: let the regular entry point report which error
        return wan_attn_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, S, H, D, nullptr, 0, stream);
    }
    if (need > static_cast<size_t>(WAN_ATTN_NOALLOC_WORKSPACE_BYTES)) return WAN_ATTN_ERR_WORKSPACE;
    void* scratch = scratch_on_current_device();
    if (!scratch) return WAN_ATTN_ERR_CUDA;
    // The dQ accumulator is zeroed and D_i fully rewritten by the backward's
    // first kernel on every call, so nothing left by an earlier call leaks in.
    return wan_attn_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, S, H, D, scratch,
                        static_cast<size_t>(WAN_ATTN_NOALLOC_WORKSPACE_BYTES), stream);
}
