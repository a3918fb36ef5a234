// internal.h -- launchers behind the C ABI and the layout workspace format.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

// Layout workspace: [header | expert_count (E) | tile_base (E x n_tiles) |
// tile_tpr (R x n_tiles) | in_rank (A = T*K, uint16)], the parts after the
// header 256-byte aligned.  Tiles are runs of at most TT consecutive tokens
// that never straddle two source ranks' token blocks, so per-rank sums are
// sums over whole tiles.  tile_base[e][j] first holds the number of expert-e
// assignments in tile j, then (after the row scan) the number in all earlier
// tiles: the stable base of tile j inside expert e's group.  in_rank[f] is the
// number of earlier assignments of f's expert inside f's tile, so
//     row(f) = expert_offsets[e] + tile_base[e][tile(t)] + in_rank[f].
// expert_count[e] is e's total.  Every word the layout reads is written
// earlier in the same call (the header's arrival counter by the tile kernel,
// before the row kernel counts on it), so a workspace needs no initialisation.
struct LayoutHeader {
    int64_t off_tile_base;     // byte offsets of the parts (so a reader needs no R)
    int64_t off_tile_tpr;
    int64_t off_expert_count;
    int64_t off_in_rank;
    int32_t magic;
    int32_t T, K, E, R;
    int32_t TT;        // tokens per tile
    int32_t tpb;       // tiles per source block
    int32_t n_tiles;   // R * tpb
    uint32_t done;     // arrival counter of the row kernel (zeroed by the tile kernel)
    int32_t pad[7];
};
static_assert(sizeof(LayoutHeader) == 96, "header layout");

constexpr int32_t kLayoutMagic = 0x4d6f4531;  // "MoE1"
constexpr int kMaxTileAssign = 2048;          // TT * K <= this (64 warp chunks)
constexpr int kMaxTileChunks = kMaxTileAssign / 32;

struct Geometry {
    int TT, tpb, n_tiles;
};

// Tile geometry: about one tile per SM of a 148-SM B200 (the layout kernel
// runs one 1024-thread CTA per tile), at least kMinTileAssign and at most
// kMaxTileAssign assignments per tile.  A pure function of the sizes, so the
// workspace size is known before any device is touched.
constexpr int kMinTileAssign = 512;            // small problems: fewer, fuller tiles

inline Geometry layout_geometry(int T, int K, int R) {
    const int Tb = R > 0 ? T / R : 0;
    int per_block = R > 0 ? 148 / R : 1;          // tiles per source block, <= 148 in all
    // No more tiles than it takes to give each at least kMinTileAssign
    // assignments: a small problem then launches fewer, fuller CTAs and its
    // rows of per-tile counts are shorter (measured: Mixtral-shaped layout
    // 14.3 -> 12.7 us; unchanged for the large shapes).
    const int64_t want = ((int64_t)Tb * K + kMinTileAssign - 1) / kMinTileAssign;
    if (want < per_block) per_block = (int)want;
    if (per_block < 1) per_block = 1;
    int tt = (Tb + per_block - 1) / per_block;
    int cap = kMaxTileAssign / K;
    if (tt > cap) tt = cap;
    if (tt < 1) tt = 1;
    if (Tb > 0 && tt > Tb) tt = Tb;
    Geometry g;
    g.TT = tt;
    g.tpb = Tb > 0 ? (Tb + tt - 1) / tt : 0;
    g.n_tiles = R * g.tpb;
    return g;
}

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// The ring permute (fan-out K <= 2): one CTA per SM streams a contiguous
// range of 4 KB row pieces through shared-memory buffers filled by bulk
// loads.  A CTA's table holds the rows of at most kRingRows (token, slot)
// pairs; every mbarrier wait gives up after kRingSpinLimit probes.
constexpr int kRingPiece = 4096;
constexpr int kRingRows = 2048;
constexpr unsigned kRingSpinLimit = 1u << 22;

// The claim the direct expert-parallel dispatch records for a row of a
// receive buffer: the sending rank (< 64) and its flat index f = t*K + k
// (< 2^25) in one non-negative int32; -1 marks a row nobody holds.
constexpr int kClaimShift = 25;
__host__ __device__ inline int32_t claim_code(int rank, int64_t f) {
    return (int32_t)(((uint32_t)rank << kClaimShift) | (uint32_t)f);
}

struct WsLayout {
    size_t expert_count, tile_base, tile_tpr, in_rank, total;
};

inline WsLayout workspace_layout(int E, int R, int n_tiles, int64_t A) {
    WsLayout w;
    w.expert_count = align256(sizeof(LayoutHeader));
    w.tile_base = align256(w.expert_count + sizeof(int32_t) * (size_t)E);
    w.tile_tpr = w.tile_base + align256(sizeof(int32_t) * (size_t)E * (size_t)n_tiles);
    w.in_rank = w.tile_tpr + align256(sizeof(int32_t) * (size_t)n_tiles * (size_t)R);
    w.total = w.in_rank + align256(sizeof(uint16_t) * (size_t)A);
    return w;
}

int sm_count_current_device();

// MOE_OK for cudaSuccess; otherwise records err for moe_last_cuda_error
// (per host thread) and returns MOE_ERR_CUDA.
int cuda_result(cudaError_t err);

cudaError_t launch_layout(const int64_t* topk_idx, int T, int K, int E, int R, int align,
                          int32_t* tokens_per_expert, int32_t* counts, int32_t* splits,
                          int32_t* tokens_per_rank, uint8_t* is_token_in_rank,
                          int32_t* expert_offsets, void* workspace, int32_t* status,
                          cudaStream_t stream);

cudaError_t launch_permute(const uint16_t* x, const int64_t* topk_idx, int T, int K, int E, int H,
                           const int32_t* expert_offsets, const void* workspace, int zero_pad,
                           int64_t N_cap, uint16_t* x_perm, int32_t* row_to_flat,
                           int32_t* flat_to_row, int32_t* status, cudaStream_t stream);

cudaError_t launch_permute_payload(const void* x, int64_t row_bytes, const void* aux,
                                   int64_t aux_row_bytes, const int64_t* topk_idx, int T, int K,
                                   int E, const int32_t* expert_offsets, const void* workspace,
                                   int zero_pad, int64_t N_cap, void* x_perm, void* aux_perm,
                                   int32_t* row_to_flat, int32_t* flat_to_row, int32_t* status,
                                   cudaStream_t stream);

cudaError_t launch_expert_scale(const uint16_t* rows, int64_t N_cap, const int32_t* expert_offsets,
                                const int32_t* tokens_per_expert, int E, int H,
                                const float* scales, uint16_t* out, int32_t* status,
                                cudaStream_t stream);

cudaError_t launch_combine(const uint16_t* rows, int64_t N_cap, const int32_t* row_to_flat,
                           const int32_t* flat_to_row, const void* weights, int weight_dtype,
                           int T, int K, int H, int validate, uint16_t* out, int32_t* status,
                           cudaStream_t stream);

cudaError_t launch_combine_f32(const float* rows, int64_t N_cap, const int32_t* row_to_flat,
                               const int32_t* flat_to_row, const void* weights, int weight_dtype,
                               int T, int K, int H, int validate, float* out, int32_t* status,
                               cudaStream_t stream);

cudaError_t launch_combine_backward_f32(const float* grad_out, const float* rows, int64_t N_cap,
                                        const int32_t* row_to_flat, const int32_t* flat_to_row,
                                        const void* weights, int weight_dtype, int T, int K, int H,
                                        const int32_t* expert_offsets, int E, int zero_pad,
                                        float* grad_rows, void* grad_weights, int32_t* status,
                                        cudaStream_t stream);

cudaError_t launch_scatter_flat_index(const int32_t* row_flat, int64_t N, int T, int K,
                                      int32_t* flat_to_row, int32_t* status, cudaStream_t stream);

cudaError_t launch_permute_to_ranks(const uint16_t* x, const int64_t* topk_idx, int T, int K,
                                    int E, int R, int H, const int32_t* dest_base,
                                    const void* workspace, uint16_t* const* dest_rows,
                                    int32_t* const* dest_claims, int64_t dest_cap, int rank,
                                    const int32_t* own_offsets, const int32_t* own_counts,
                                    int zero_pad, int32_t* flat_to_row, int32_t* status,
                                    cudaStream_t stream);

cudaError_t launch_combine_from_ranks(const uint16_t* const* rows, const int32_t* const* claims,
                                      int R, int rank, int64_t N_cap, const int32_t* flat_to_row,
                                      const int64_t* topk_idx, int E, const void* weights,
                                      int weight_dtype, int T, int K, int H, uint16_t* out,
                                      int32_t* status, cudaStream_t stream);

cudaError_t launch_rank_bases(const int32_t* all_counts, int R, int E, int rank, int align,
                              int32_t* dest_base, int32_t* own_offsets, int32_t* own_counts,
                              int32_t* max_rows, int32_t* status, cudaStream_t stream);

cudaError_t launch_combine_slots_from_ranks(const uint16_t* const* rows,
                                            const int32_t* const* claims, int R, int rank,
                                            int64_t N_cap, const int32_t* flat_to_row,
                                            const int64_t* topk_idx, int E, const void* weights,
                                            int weight_dtype, int T, int K, int H, uint16_t* out,
                                            int32_t* status, cudaStream_t stream);

cudaError_t launch_segment_labels(const int32_t* counts, int n, int modulo, int64_t rows,
                                  int64_t* labels, int32_t* status, cudaStream_t stream);

cudaError_t launch_combine_backward(const uint16_t* grad_out, const uint16_t* rows, int64_t N_cap,
                                    const int32_t* row_to_flat, const int32_t* flat_to_row,
                                    const void* weights, int weight_dtype, int T, int K, int H,
                                    const int32_t* expert_offsets, int E, int zero_pad,
                                    uint16_t* grad_rows, void* grad_weights, int32_t* status,
                                    cudaStream_t stream);

}  // namespace moe
