// layout_noalloc.cu -- the routing layout for callers that cannot allocate
// device memory.
//
// moe_dispatch_layout needs a caller-provided workspace.  Some callers have
// no way to provide one: code that runs while another component owns every
// byte of the device's memory pool (an inference server's plugin, a
// framework operator that only receives the tensors it is handed), and hot
// paths where cudaMalloc/cudaFree must not run because they can synchronise
// the whole device.  For them this file keeps the workspace in a file-scope
// device array that exists, once per GPU, from the moment the library is
// loaded until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "moe_dispatch.h"

namespace {

// The shared scratch.  In host code this name is only a host-side stand-in
// for the device array (its address is not a device address), so the host
// asks the runtime for the device address and passes that to the kernels.
static __device__ __align__(256) unsigned char g_layout_scratch[MOE_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mutex;
void* g_scratch_ptr[64] = {};

// Device address of g_layout_scratch on the current device, looked up once
// per device (with that device current) and cached for the life of the
// process.  The address belongs to the device's context at that first
// call; cudaDeviceReset destroys it, after which this entry point is not
// supported in the process (documented in the header).
int scratch_on_current_device(void** out) {
    int dev = -1;
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return moe::cuda_result(e);
    if (dev < 0 || dev >= 64) return moe::cuda_result(cudaErrorInvalidDevice);
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        const cudaError_t e2 = cudaGetSymbolAddress(&p, g_layout_scratch);
        if (e2 != cudaSuccess) return moe::cuda_result(e2);
        if (p == nullptr) return moe::cuda_result(cudaErrorInvalidSymbol);
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" int moe_dispatch_layout_noalloc(const int64_t* topk_idx, int T, int K, int E, int R,
                                           int align, int32_t* tokens_per_expert, int32_t* counts,
                                           int32_t* splits, int32_t* tokens_per_rank,
                                           uint8_t* is_token_in_rank, int32_t* expert_offsets,
                                           int32_t* status, cudaStream_t stream) {
    const size_t need = moe_layout_workspace_bytes(T, K, E, R);
    if (need == 0) return MOE_ERR_INVALID_ARG;
    if (need > (size_t)MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_SCRATCH;
    void* ws = nullptr;
    const int rc = scratch_on_current_device(&ws);
    if (rc != MOE_OK) return rc;
    // What must start at zero (the row kernel's arrival counter) is zeroed
    // by the layout's first kernel, and its kernels write every other word
    // they read before reading it, so the scratch left by an earlier call
    // needs no clearing here.
    return moe_dispatch_layout(topk_idx, T, K, E, R, align, tokens_per_expert, counts, splits,
                               tokens_per_rank, is_token_in_rank, expert_offsets, ws, status,
                               stream);
}
