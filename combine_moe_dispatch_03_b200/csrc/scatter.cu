// scatter.cu -- the scatter step of the folded restore: flat_to_row from the
// flat index (token * top_k + slot) each gathered row holds, with the
// coverage check.  Source: DeepSpeed PR "AutoEP: support
// combine_impl=fused_weighted_sum with AutoEP+AutoTP folding", Change: the
// folded path gathers one flat index per row instead of token and slot,
// scatters the routing data into [tokens, top_k], and "raises a clear
// RuntimeError if the gathered rows do not cover every (token, slot)".
//
// Three stream-ordered steps: flat_to_row <- -1 (memset), then every row
// claims its flat index with an atomic compare-and-swap (a second claim is a
// duplicate), then every (token, slot) must have been claimed.
#include "common.cuh"
#include "internal.h"

namespace moe {

__global__ void __launch_bounds__(kBlock)
scatter_claim_kernel(const int32_t* __restrict__ row_flat, int64_t N, int64_t A,
                     int32_t* __restrict__ f2r, int32_t* __restrict__ status) {
    int bad = 0;
    const int64_t stride = (int64_t)gridDim.x * kBlock;
    for (int64_t row = (int64_t)blockIdx.x * kBlock + threadIdx.x; row < N; row += stride) {
        const int32_t f = row_flat[row];
        if (f == -1) continue;
        if (f < 0 || (int64_t)f >= A) {
            bad |= MOE_ST_COVERAGE;
            continue;
        }
        if (atomicCAS(f2r + f, -1, (int32_t)row) != -1) bad |= MOE_ST_COVERAGE;
    }
    warp_status_or(status, bad);
}

__global__ void __launch_bounds__(kBlock)
scatter_check_kernel(const int32_t* __restrict__ f2r, int64_t A, int32_t* __restrict__ status) {
    int bad = 0;
    const int64_t stride = (int64_t)gridDim.x * kBlock;
    for (int64_t f = (int64_t)blockIdx.x * kBlock + threadIdx.x; f < A; f += stride)
        if (f2r[f] < 0) bad |= MOE_ST_COVERAGE;
    warp_status_or(status, bad);
}

cudaError_t launch_scatter_flat_index(const int32_t* row_flat, int64_t N, int T, int K,
                                      int32_t* flat_to_row, int32_t* status, cudaStream_t stream) {
    const int64_t A = (int64_t)T * K;
    if (A > 0) {
        cudaError_t err = cudaMemsetAsync(flat_to_row, 0xFF, sizeof(int32_t) * (size_t)A, stream);
        if (err != cudaSuccess) return err;
    }
    const int cap = sm_count_current_device() * 8;
    int64_t g1 = (N + kBlock - 1) / kBlock;
    if (g1 > cap) g1 = cap;
    if (g1 < 1) g1 = 1;
    scatter_claim_kernel<<<(int)g1, kBlock, 0, stream>>>(row_flat, N, A, flat_to_row, status);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    int64_t g2 = (A + kBlock - 1) / kBlock;
    if (g2 > cap) g2 = cap;
    if (g2 < 1) g2 = 1;
    scatter_check_kernel<<<(int)g2, kBlock, 0, stream>>>(flat_to_row, A, status);
    return cudaGetLastError();
}

}  // namespace moe
