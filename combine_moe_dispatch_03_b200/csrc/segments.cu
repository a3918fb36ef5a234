// segments.cu -- row labels from segment counts: the receive side of expert
// parallelism.  After the payload all-to-all a rank holds, from every source
// rank s in turn, received_counts[s][e] rows for each of its local experts e
// in local-expert order (DeepSpeed PR "Derive AutoEP rank splits from the
// per-expert count exchange": received_counts[s, e] is the number of tokens
// source rank s sends to local expert e).  Labelling every received row with
// its local expert turns the regrouping by expert into an ordinary layout +
// permute with top_k = 1.
//
// Row i of a buffer of n consecutive segments, segment j holding counts[j]
// rows, gets label j % modulo (for the received buffer, j = s * E_local + e
// and modulo = E_local).  One grid-stride kernel: every CTA scans the <= 1024
// counts in shared memory, then each row finds its segment by binary search.
#include "common.cuh"
#include "internal.h"

namespace moe {

__global__ void __launch_bounds__(kBlock)
segment_labels_kernel(const int32_t* __restrict__ counts, int n, int modulo, int64_t rows,
                      int64_t* __restrict__ labels, int32_t* __restrict__ status) {
    __shared__ int pre[MOE_MAX_E + 1];
    __shared__ int scratch[kWarps + 1];
    const int tid = threadIdx.x;
    pdl_wait();
    pdl_trigger();
    int bad = 0;
    for (int j = tid; j < n; j += kBlock) {
        const int c = counts[j];
        if (c < 0) bad |= MOE_ST_COVERAGE;
        pre[j] = c > 0 ? c : 0;
    }
    __syncthreads();
    const int total = block_exclusive_scan<MOE_MAX_E / kBlock>(pre, n, scratch);
    if (tid == 0) pre[n] = total;
    __syncthreads();
    if (blockIdx.x == 0 && tid == 0 && (int64_t)total > rows) bad |= MOE_ST_CAPACITY;
    const int64_t stride = (int64_t)gridDim.x * kBlock;
    for (int64_t i = (int64_t)blockIdx.x * kBlock + tid; i < rows; i += stride) {
        if (i >= (int64_t)total) {
            labels[i] = -1;
            continue;
        }
        // Largest j with pre[j] <= i: an empty segment shares its start with
        // the next one, and the later (non-empty) one wins.
        const int j = upper_index(pre, n + 1, (int)i);
        labels[i] = (int64_t)(j % modulo);
    }
    warp_status_or(status, bad);
}

cudaError_t launch_segment_labels(const int32_t* counts, int n, int modulo, int64_t rows,
                                  int64_t* labels, int32_t* status, cudaStream_t stream) {
    int64_t grid = (rows + kBlock - 1) / kBlock;
    const int cap = sm_count_current_device() * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    return launch_pdl(segment_labels_kernel, dim3((int)grid), dim3(kBlock), 0, stream, counts, n,
                      modulo, rows, labels, status);
}

}  // namespace moe
