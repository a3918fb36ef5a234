// capi.cu -- the extern "C" entry points of libmoe_dispatch.so: argument
// checks on the host, then kernel launches on the caller's stream.  No call
// allocates, synchronises or reads device memory on the host.  Every call
// that enqueues work is an NVTX range named after the call, so a profiler
// timeline shows which kernels each call launched (header-only NVTX: without
// a tool attached a range costs a branch).
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <atomic>

#include "internal.h"
#include "moe_dispatch.h"

namespace moe {

// Per-device SM count (the only state kept between calls).
int sm_count_current_device() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < 64) {
        int v = cache[dev].load(std::memory_order_relaxed);
        if (v > 0) return v;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

// The CUDA error behind the calling thread's last MOE_ERR_CUDA.
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

int cuda_result(cudaError_t err) {
    if (err == cudaSuccess) return MOE_OK;
    g_last_cuda_error = err;
    return MOE_ERR_CUDA;
}

}  // namespace moe

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Sizes shared by the calls; see the limits in moe_dispatch.h.
bool sizes_ok(int T, int K, int E) {
    if (T < 0 || K < 1 || K > MOE_MAX_K || E < 1 || E > MOE_MAX_E) return false;
    if ((int64_t)T * K > INT32_MAX) return false;
    return true;
}

bool hidden_ok(int H) { return H > 0 && (H % 8) == 0; }

bool ncap_ok(int64_t N_cap, int T, int K) {
    return N_cap >= (int64_t)T * K && N_cap <= INT32_MAX;
}

int finish(cudaError_t err) { return moe::cuda_result(err); }

struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

}  // namespace

extern "C" {

size_t moe_layout_workspace_bytes(int T, int K, int E, int R) {
    if (!sizes_ok(T, K, E) || R < 1 || R > MOE_MAX_R || E % R || T % R) return 0;
    const moe::Geometry g = moe::layout_geometry(T, K, R);
    return moe::workspace_layout(E, R, g.n_tiles, (int64_t)T * K).total;
}

int64_t moe_worst_case_rows(int T, int K, int E, int align) {
    if (!sizes_ok(T, K, E) || align < 1) return -1;
    return (int64_t)T * K + (int64_t)E * (align - 1);
}

int moe_dispatch_layout(const int64_t* topk_idx, int T, int K, int E, int R, int align,
                        int32_t* tokens_per_expert, int32_t* counts, int32_t* splits,
                        int32_t* tokens_per_rank, uint8_t* is_token_in_rank,
                        int32_t* expert_offsets, void* workspace, int32_t* status,
                        cudaStream_t stream) {
    NvtxRange range("moe_dispatch_layout");
    if (!sizes_ok(T, K, E) || R < 1 || R > MOE_MAX_R || E % R || T % R || align < 1)
        return MOE_ERR_INVALID_ARG;
    if ((int64_t)T * K + (int64_t)E * (align - 1) > INT32_MAX) return MOE_ERR_INVALID_ARG;
    if (!tokens_per_expert || !counts || !splits || !tokens_per_rank || !expert_offsets ||
        !workspace || !status)
        return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!topk_idx || !is_token_in_rank)) return MOE_ERR_INVALID_ARG;
    if (!aligned(topk_idx, 8) || !aligned(workspace, 16) || !aligned(tokens_per_expert, 4) ||
        !aligned(counts, 4) || !aligned(splits, 4) || !aligned(tokens_per_rank, 4) ||
        !aligned(expert_offsets, 4) || !aligned(status, 4))
        return MOE_ERR_INVALID_ARG;
    return finish(moe::launch_layout(topk_idx, T, K, E, R, align, tokens_per_expert, counts,
                                     splits, tokens_per_rank, is_token_in_rank, expert_offsets,
                                     workspace, status, stream));
}

int moe_permute(const uint16_t* x, const int64_t* topk_idx, int T, int K, int E, int H,
                const int32_t* expert_offsets, const void* workspace, int zero_pad,
                int64_t N_cap, uint16_t* x_perm, int32_t* row_to_flat, int32_t* flat_to_row,
                int32_t* status, cudaStream_t stream) {
    NvtxRange range("moe_permute");
    if (!sizes_ok(T, K, E) || !hidden_ok(H) || !ncap_ok(N_cap, T, K)) return MOE_ERR_INVALID_ARG;
    if (!expert_offsets || !workspace || !status) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !topk_idx || !flat_to_row)) return MOE_ERR_INVALID_ARG;
    if (N_cap > 0 && (!x_perm || !row_to_flat)) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(x_perm, 16) || !aligned(topk_idx, 8) ||
        !aligned(workspace, 16) || !aligned(expert_offsets, 4) || !aligned(row_to_flat, 4) ||
        !aligned(flat_to_row, 4) || !aligned(status, 4))
        return MOE_ERR_INVALID_ARG;
    return finish(moe::launch_permute(x, topk_idx, T, K, E, H, expert_offsets, workspace,
                                      zero_pad, N_cap, x_perm, row_to_flat, flat_to_row, status,
                                      stream));
}

int moe_dispatch(const uint16_t* x, const int64_t* topk_idx, int T, int K, int E, int R, int H,
                 int align, int32_t* tokens_per_expert, int32_t* counts, int32_t* splits,
                 int32_t* tokens_per_rank, uint8_t* is_token_in_rank, int32_t* expert_offsets,
                 void* workspace, int zero_pad, int64_t N_cap, uint16_t* x_perm,
                 int32_t* row_to_flat, int32_t* flat_to_row, int32_t* status,
                 cudaStream_t stream) {
    NvtxRange range("moe_dispatch");
    // Every check of both calls, before anything is enqueued.
    if (!sizes_ok(T, K, E) || R < 1 || R > MOE_MAX_R || E % R || T % R || align < 1 ||
        !hidden_ok(H) || !ncap_ok(N_cap, T, K))
        return MOE_ERR_INVALID_ARG;
    if ((int64_t)T * K + (int64_t)E * (align - 1) > INT32_MAX) return MOE_ERR_INVALID_ARG;
    if (!tokens_per_expert || !counts || !splits || !tokens_per_rank || !expert_offsets ||
        !workspace || !status)
        return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !topk_idx || !is_token_in_rank || !flat_to_row)) return MOE_ERR_INVALID_ARG;
    if (N_cap > 0 && (!x_perm || !row_to_flat)) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(x_perm, 16) || !aligned(topk_idx, 8) ||
        !aligned(workspace, 16) || !aligned(tokens_per_expert, 4) || !aligned(counts, 4) ||
        !aligned(splits, 4) || !aligned(tokens_per_rank, 4) || !aligned(expert_offsets, 4) ||
        !aligned(row_to_flat, 4) || !aligned(flat_to_row, 4) || !aligned(status, 4))
        return MOE_ERR_INVALID_ARG;
    const cudaError_t e = moe::launch_layout(topk_idx, T, K, E, R, align, tokens_per_expert,
                                             counts, splits, tokens_per_rank, is_token_in_rank,
                                             expert_offsets, workspace, status, stream);
    if (e != cudaSuccess) return finish(e);
    return finish(moe::launch_permute(x, topk_idx, T, K, E, H, expert_offsets, workspace,
                                      zero_pad, N_cap, x_perm, row_to_flat, flat_to_row, status,
                                      stream));
}

int moe_expert_scale(const uint16_t* rows, int64_t N_cap, const int32_t* expert_offsets,
                     const int32_t* tokens_per_expert, int E, int H, const float* scales,
                     uint16_t* out, int32_t* status, cudaStream_t stream) {
    NvtxRange range("moe_expert_scale");
    if (E < 1 || E > MOE_MAX_E || !hidden_ok(H) || N_cap < 0 || N_cap > INT32_MAX)
        return MOE_ERR_INVALID_ARG;
    if (!expert_offsets || !tokens_per_expert || !scales || !status) return MOE_ERR_INVALID_ARG;
    if (N_cap > 0 && (!rows || !out)) return MOE_ERR_INVALID_ARG;
    if (N_cap > 0 && rows == out) return MOE_ERR_INVALID_ARG;
    if (!aligned(rows, 16) || !aligned(out, 16) || !aligned(expert_offsets, 4) ||
        !aligned(tokens_per_expert, 4) || !aligned(scales, 4) || !aligned(status, 4))
        return MOE_ERR_INVALID_ARG;
    return finish(moe::launch_expert_scale(rows, N_cap, expert_offsets, tokens_per_expert, E, H,
                                           scales, out, status, stream));
}

int moe_combine_weighted(const uint16_t* rows, int64_t N_cap, const int32_t* row_to_flat,
                         const int32_t* flat_to_row, const void* weights, int weight_dtype,
                         int T, int K, int H, int validate, uint16_t* out, int32_t* status,
                         cudaStream_t stream) {
    NvtxRange range("moe_combine_weighted");
    if (T < 0 || K < 1 || K > MOE_MAX_K || (int64_t)T * K > INT32_MAX || !hidden_ok(H) ||
        N_cap < 0 || N_cap > INT32_MAX)
        return MOE_ERR_INVALID_ARG;
    if (weight_dtype != MOE_DTYPE_F32 && weight_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    if (!status) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!flat_to_row || !out)) return MOE_ERR_INVALID_ARG;
    if (T > 0 && N_cap > 0 && !rows) return MOE_ERR_INVALID_ARG;
    if (validate && N_cap > 0 && !row_to_flat) return MOE_ERR_INVALID_ARG;
    const size_t wal = weight_dtype == MOE_DTYPE_F32 ? 4 : 2;
    if (!aligned(rows, 16) || !aligned(out, 16) || !aligned(flat_to_row, 4) ||
        !aligned(row_to_flat, 4) || !aligned(weights, wal) || !aligned(status, 4))
        return MOE_ERR_INVALID_ARG;
    if (T == 0 && !validate) return MOE_OK;
    return finish(moe::launch_combine(rows, N_cap, row_to_flat, flat_to_row, weights, weight_dtype,
                                      T, K, H, validate, out, status, stream));
}

int moe_combine_backward(const uint16_t* grad_out, const uint16_t* rows, int64_t N_cap,
                         const int32_t* row_to_flat, const int32_t* flat_to_row,
                         const void* weights, int weight_dtype, int T, int K, int H,
                         const int32_t* expert_offsets, int E, int zero_pad,
                         uint16_t* grad_rows, void* grad_weights, int32_t* status,
                         cudaStream_t stream) {
    NvtxRange range("moe_combine_backward");
    if (T < 0 || K < 1 || K > MOE_MAX_K || (int64_t)T * K > INT32_MAX || !hidden_ok(H) ||
        N_cap < 0 || N_cap > INT32_MAX || E < 1 || E > MOE_MAX_E)
        return MOE_ERR_INVALID_ARG;
    if (weight_dtype != MOE_DTYPE_F32 && weight_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    if (!status || !expert_offsets) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!grad_out || !flat_to_row || !weights)) return MOE_ERR_INVALID_ARG;
    if (N_cap > 0 && (!rows || !grad_rows)) return MOE_ERR_INVALID_ARG;
    if (zero_pad && N_cap > 0 && !row_to_flat) return MOE_ERR_INVALID_ARG;
    const size_t wal = weight_dtype == MOE_DTYPE_F32 ? 4 : 2;
    if (!aligned(grad_out, 16) || !aligned(rows, 16) || !aligned(grad_rows, 16) ||
        !aligned(flat_to_row, 4) || !aligned(row_to_flat, 4) || !aligned(weights, wal) ||
        !aligned(grad_weights, wal) || !aligned(expert_offsets, 4) || !aligned(status, 4))
        return MOE_ERR_INVALID_ARG;
    if (T == 0 && !zero_pad) return MOE_OK;
    return finish(moe::launch_combine_backward(grad_out, rows, N_cap, row_to_flat, flat_to_row,
                                               weights, weight_dtype, T, K, H, expert_offsets, E,
                                               zero_pad, grad_rows, grad_weights, status, stream));
}

int moe_permute_payload(const void* x, int64_t row_bytes, const void* aux, int64_t aux_row_bytes,
                        const int64_t* topk_idx, int T, int K, int E,
                        const int32_t* expert_offsets, const void* workspace, int zero_pad,
                        int64_t N_cap, void* x_perm, void* aux_perm, int32_t* row_to_flat,
                        int32_t* flat_to_row, int32_t* status, cudaStream_t stream) {
    NvtxRange range("moe_permute_payload");
    if (!sizes_ok(T, K, E) || !ncap_ok(N_cap, T, K)) return MOE_ERR_INVALID_ARG;
    if (row_bytes <= 0 || row_bytes % 16 || row_bytes / 16 > INT32_MAX / 2) return MOE_ERR_INVALID_ARG;
    if (aux_row_bytes < 0 || aux_row_bytes % 4 || aux_row_bytes > 65536) return MOE_ERR_INVALID_ARG;
    if (aux_row_bytes > 0 && ((T > 0 && !aux) || (N_cap > 0 && !aux_perm))) return MOE_ERR_INVALID_ARG;
    if (!expert_offsets || !workspace || !status) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !topk_idx || !flat_to_row)) return MOE_ERR_INVALID_ARG;
    if (N_cap > 0 && (!x_perm || !row_to_flat)) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(x_perm, 16) || !aligned(aux, 4) || !aligned(aux_perm, 4) ||
        !aligned(topk_idx, 8) || !aligned(workspace, 16) || !aligned(expert_offsets, 4) ||
        !aligned(row_to_flat, 4) || !aligned(flat_to_row, 4) || !aligned(status, 4))
        return MOE_ERR_INVALID_ARG;
    return finish(moe::launch_permute_payload(x, row_bytes, aux, aux_row_bytes, topk_idx, T, K, E,
                                              expert_offsets, workspace, zero_pad, N_cap, x_perm,
                                              aux_perm, row_to_flat, flat_to_row, status, stream));
}

int moe_combine_weighted_f32(const float* rows, int64_t N_cap, const int32_t* row_to_flat,
                             const int32_t* flat_to_row, const void* weights, int weight_dtype,
                             int T, int K, int H, int validate, float* out, int32_t* status,
                             cudaStream_t stream) {
    NvtxRange range("moe_combine_weighted_f32");
    if (T < 0 || K < 1 || K > MOE_MAX_K || (int64_t)T * K > INT32_MAX || H <= 0 || H % 4 ||
        N_cap < 0 || N_cap > INT32_MAX)
        return MOE_ERR_INVALID_ARG;
    if (weight_dtype != MOE_DTYPE_F32 && weight_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    if (!status) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!flat_to_row || !out)) return MOE_ERR_INVALID_ARG;
    if (T > 0 && N_cap > 0 && !rows) return MOE_ERR_INVALID_ARG;
    if (validate && N_cap > 0 && !row_to_flat) return MOE_ERR_INVALID_ARG;
    const size_t wal = weight_dtype == MOE_DTYPE_F32 ? 4 : 2;
    if (!aligned(rows, 16) || !aligned(out, 16) || !aligned(flat_to_row, 4) ||
        !aligned(row_to_flat, 4) || !aligned(weights, wal) || !aligned(status, 4))
        return MOE_ERR_INVALID_ARG;
    if (T == 0 && !validate) return MOE_OK;
    return finish(moe::launch_combine_f32(rows, N_cap, row_to_flat, flat_to_row, weights,
                                          weight_dtype, T, K, H, validate, out, status, stream));
}

int moe_combine_backward_f32(const float* grad_out, const float* rows, int64_t N_cap,
                             const int32_t* row_to_flat, const int32_t* flat_to_row,
                             const void* weights, int weight_dtype, int T, int K, int H,
                             const int32_t* expert_offsets, int E, int zero_pad,
                             float* grad_rows, void* grad_weights, int32_t* status,
                             cudaStream_t stream) {
    NvtxRange range("moe_combine_backward_f32");
    if (T < 0 || K < 1 || K > MOE_MAX_K || (int64_t)T * K > INT32_MAX || H <= 0 || H % 4 ||
        N_cap < 0 || N_cap > INT32_MAX || E < 1 || E > MOE_MAX_E)
        return MOE_ERR_INVALID_ARG;
    if (weight_dtype != MOE_DTYPE_F32 && weight_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    if (!status || !expert_offsets) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!grad_out || !flat_to_row || !weights)) return MOE_ERR_INVALID_ARG;
    if (N_cap > 0 && (!rows || !grad_rows)) return MOE_ERR_INVALID_ARG;
    if (zero_pad && N_cap > 0 && !row_to_flat) return MOE_ERR_INVALID_ARG;
    const size_t wal = weight_dtype == MOE_DTYPE_F32 ? 4 : 2;
    if (!aligned(grad_out, 16) || !aligned(rows, 16) || !aligned(grad_rows, 16) ||
        !aligned(flat_to_row, 4) || !aligned(row_to_flat, 4) || !aligned(weights, wal) ||
        !aligned(grad_weights, wal) || !aligned(expert_offsets, 4) || !aligned(status, 4))
        return MOE_ERR_INVALID_ARG;
    if (T == 0 && !zero_pad) return MOE_OK;
    return finish(moe::launch_combine_backward_f32(grad_out, rows, N_cap, row_to_flat, flat_to_row,
                                                   weights, weight_dtype, T, K, H, expert_offsets,
                                                   E, zero_pad, grad_rows, grad_weights, status,
                                                   stream));
}

int moe_scatter_flat_index(const int32_t* row_flat, int64_t N, int T, int K,
                           int32_t* flat_to_row, int32_t* status, cudaStream_t stream) {
    NvtxRange range("moe_scatter_flat_index");
    if (T < 0 || K < 1 || K > MOE_MAX_K || (int64_t)T * K > INT32_MAX || N < 0 || N > INT32_MAX)
        return MOE_ERR_INVALID_ARG;
    if (!status || (N > 0 && !row_flat) || (T > 0 && !flat_to_row)) return MOE_ERR_INVALID_ARG;
    if (!aligned(row_flat, 4) || !aligned(flat_to_row, 4) || !aligned(status, 4))
        return MOE_ERR_INVALID_ARG;
    return finish(moe::launch_scatter_flat_index(row_flat, N, T, K, flat_to_row, status, stream));
}

int moe_segment_labels(const int32_t* counts, int n, int modulo, int64_t rows, int64_t* labels,
                       int32_t* status, cudaStream_t stream) {
    NvtxRange range("moe_segment_labels");
    if (n < 1 || n > MOE_MAX_E || modulo < 1 || rows < 0 || rows > INT32_MAX)
        return MOE_ERR_INVALID_ARG;
    if (!counts || !status || (rows > 0 && !labels)) return MOE_ERR_INVALID_ARG;
    if (!aligned(counts, 4) || !aligned(labels, 8) || !aligned(status, 4))
        return MOE_ERR_INVALID_ARG;
    return finish(moe::launch_segment_labels(counts, n, modulo, rows, labels, status, stream));
}

int moe_rank_bases(const int32_t* all_counts, int R, int E, int rank, int align,
                   int32_t* dest_base, int32_t* own_offsets, int32_t* own_counts,
                   int32_t* max_rows, int32_t* status, cudaStream_t stream) {
    NvtxRange range("moe_rank_bases");
    if (R < 1 || R > MOE_MAX_R || E < 1 || E > MOE_MAX_E || E % R || rank < 0 || rank >= R ||
        align < 1)
        return MOE_ERR_INVALID_ARG;
    if (!all_counts || !dest_base || !own_offsets || !own_counts || !max_rows || !status)
        return MOE_ERR_INVALID_ARG;
    if (!aligned(all_counts, 4) || !aligned(dest_base, 4) || !aligned(own_offsets, 4) ||
        !aligned(own_counts, 4) || !aligned(max_rows, 4) || !aligned(status, 4))
        return MOE_ERR_INVALID_ARG;
    return finish(moe::launch_rank_bases(all_counts, R, E, rank, align, dest_base, own_offsets,
                                         own_counts, max_rows, status, stream));
}

int moe_permute_to_ranks(const uint16_t* x, const int64_t* topk_idx, int T, int K, int E, int R,
                         int H, const int32_t* dest_base, const void* workspace,
                         uint16_t* const* dest_rows, int32_t* const* dest_claims,
                         int64_t dest_cap, int rank, const int32_t* own_offsets,
                         const int32_t* own_counts, int zero_pad, int32_t* flat_to_row,
                         int32_t* status, cudaStream_t stream) {
    NvtxRange range("moe_permute_to_ranks");
    if (!sizes_ok(T, K, E) || !hidden_ok(H) || R < 1 || R > MOE_MAX_R || E % R || rank < 0 ||
        rank >= R || dest_cap < 0 || dest_cap > INT32_MAX)
        return MOE_ERR_INVALID_ARG;
    if (dest_claims && ((int64_t)T * K > (int64_t(1) << moe::kClaimShift) ||
                        !aligned(dest_claims, 8)))
        return MOE_ERR_INVALID_ARG;
    if (!dest_base || !workspace || !dest_rows || !own_offsets || !own_counts || !status)
        return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !topk_idx || !flat_to_row)) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(topk_idx, 8) || !aligned(workspace, 16) ||
        !aligned(dest_rows, 8) || !aligned(dest_base, 4) || !aligned(own_offsets, 4) ||
        !aligned(own_counts, 4) || !aligned(flat_to_row, 4) || !aligned(status, 4))
        return MOE_ERR_INVALID_ARG;
    return finish(moe::launch_permute_to_ranks(x, topk_idx, T, K, E, R, H, dest_base, workspace,
                                               dest_rows, dest_claims, dest_cap, rank, own_offsets,
                                               own_counts, zero_pad, flat_to_row, status, stream));
}

int moe_combine_from_ranks(const uint16_t* const* rows, const int32_t* const* claims, int R,
                           int rank, int64_t N_cap, const int32_t* flat_to_row,
                           const int64_t* topk_idx, int E, const void* weights, int weight_dtype,
                           int T, int K, int H, uint16_t* out, int32_t* status,
                           cudaStream_t stream) {
    NvtxRange range("moe_combine_from_ranks");
    if (!sizes_ok(T, K, E) || !hidden_ok(H) || R < 1 || R > MOE_MAX_R || E % R || N_cap < 0 ||
        N_cap > INT32_MAX)
        return MOE_ERR_INVALID_ARG;
    if (claims && (rank < 0 || rank >= R || (int64_t)T * K > (int64_t(1) << moe::kClaimShift) ||
                   !aligned(claims, 8)))
        return MOE_ERR_INVALID_ARG;
    if (weight_dtype != MOE_DTYPE_F32 && weight_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    if (!status || !rows) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!flat_to_row || !topk_idx || !weights || !out)) return MOE_ERR_INVALID_ARG;
    const size_t wal = weight_dtype == MOE_DTYPE_F32 ? 4 : 2;
    if (!aligned(rows, 8) || !aligned(flat_to_row, 4) || !aligned(topk_idx, 8) ||
        !aligned(weights, wal) || !aligned(out, 16) || !aligned(status, 4))
        return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    return finish(moe::launch_combine_from_ranks(rows, claims, R, rank, N_cap, flat_to_row,
                                                 topk_idx, E, weights, weight_dtype, T, K, H, out,
                                                 status, stream));
}

const char* moe_strerror(int code) {
    switch (code) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument (null pointer, size outside the limits, or misaligned buffer)";
        case MOE_ERR_CUDA: return "CUDA launch or runtime error";
        case MOE_ERR_SCRATCH: return "sizes exceed the static scratch of moe_dispatch_layout_noalloc (MOE_NOALLOC_SCRATCH_BYTES)";
        default: return "unknown return code";
    }
}

const char* moe_status_bit_name(int bit) {
    switch (bit) {
        case MOE_ST_EXPERT_OOR: return "topk_idx entry outside [0, E)";
        case MOE_ST_CAPACITY: return "padded rows exceed the row capacity N_cap";
        case MOE_ST_ROW_OOR: return "flat_to_row entry outside [0, N_cap)";
        case MOE_ST_COVERAGE: return "row maps do not cover every (token, slot) exactly once";
        case MOE_ST_LAYOUT_MISMATCH: return "layout workspace was built for other sizes";
        case MOE_ST_TIMEOUT: return "a bounded wait in a kernel timed out (kernel returned early)";
        default: return "unknown status bit";
    }
}

const char* moe_last_cuda_error(void) {
    return moe::g_last_cuda_error == cudaSuccess ? "none" : cudaGetErrorName(moe::g_last_cuda_error);
}

const char* moe_version(void) { return "moe_dispatch 0.1.0 (sm_100a)"; }

}  // extern "C"
