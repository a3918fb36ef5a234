// layout.cu -- routing layout on the device (get_dispatch_layout of the DeepEP
// issue "Does Deepep's Dispatch/Combine Support Autograd Like PyTorch's
// all_to_all?"; the count matrix [ep_size, E_local] of the DeepSpeed PR
// "Derive AutoEP rank splits from the per-expert count exchange", Redundancy;
// the group alignment of the DeepSpeed AutoEP base PR, Attribution).
//
// Two launches, no host synchronisation:
//   layout_hist_kernel  one CTA per tile of <= TT tokens: per-expert counts of
//                       the tile (warp-aggregated shared-memory histogram),
//                       is_token_in_rank rows, distinct tokens per rank.
//   layout_scan_kernel  one warp per expert: exclusive scan of the expert's
//                       tile counts (its stable per-tile bases, read back by
//                       the permute) and its per-source-block counts; the
//                       last CTA to arrive then builds the padded offsets,
//                       splits and tokens_per_rank from the other CTAs'
//                       results (arrival counter, no waiting).
//
// Bytes: reads topk_idx once (8*A), writes [T,R] flags and O(E*tiles) ints.
#include "common.cuh"
#include "internal.h"

namespace moe {

__global__ void __launch_bounds__(kBlock)
layout_hist_kernel(const int64_t* __restrict__ topk, int T, int K, int E, int R, Geometry geo,
                   uint8_t* __restrict__ itr, char* __restrict__ ws, WsLayout wl,
                   int32_t* __restrict__ status) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    unsigned long long* tokmask = reinterpret_cast<unsigned long long*>(smem_raw);  // [TT]
    int* hist = reinterpret_cast<int*>(tokmask + geo.TT);                            // [E]

    const int j = blockIdx.x;
    const int tid = threadIdx.x;
    if (j == 0 && tid == 0) {
        LayoutHeader* h = reinterpret_cast<LayoutHeader*>(ws);
        h->off_tile_base = (int64_t)wl.tile_base;
        h->off_tile_tpr = (int64_t)wl.tile_tpr;
        h->off_expert_count = (int64_t)wl.expert_count;
        h->magic = kLayoutMagic;
        h->T = T; h->K = K; h->E = E; h->R = R;
        h->TT = geo.TT; h->tpb = geo.tpb; h->n_tiles = geo.n_tiles;
        h->done = 0u;
    }
    if (j >= geo.n_tiles) return;

    int32_t* tile_base = reinterpret_cast<int32_t*>(ws + wl.tile_base);
    int32_t* tile_tpr = reinterpret_cast<int32_t*>(ws + wl.tile_tpr);
    const int Tb = T / R, El = E / R;
    const int s = j / geo.tpb, i = j - s * geo.tpb;
    const int t0 = s * Tb + i * geo.TT;
    const int t1 = min(t0 + geo.TT, (s + 1) * Tb);
    const int ntok = t1 - t0, na = ntok * K;

    for (int e = tid; e < E; e += kBlock) hist[e] = 0;
    for (int q = tid; q < ntok; q += kBlock) tokmask[q] = 0ull;
    __syncthreads();

    int bad = 0;
    const int lane = tid & 31;
    // Every thread runs the same number of iterations, so warps stay converged
    // for __match_any_sync; lanes past the end take a key no one else has.
    for (int base = 0; base < na; base += kBlock) {
        const int a = base + tid;
        int key = -1 - lane;
        if (a < na) {
            const int64_t e = topk[(int64_t)t0 * K + a];
            if (e >= 0 && e < E) key = (int)e; else bad = MOE_ST_EXPERT_OOR;
        }
        const unsigned peers = __match_any_sync(kFull, key);
        if (key >= 0) {
            if (lane == __ffs(peers) - 1) atomicAdd(&hist[key], __popc(peers));
            atomicOr(&tokmask[a / K], 1ull << (key / El));
        }
    }
    warp_status_or(status, bad);
    __syncthreads();

    for (int e = tid; e < E; e += kBlock) tile_base[(size_t)e * geo.n_tiles + j] = hist[e];
    uint8_t* itr_tile = itr + (size_t)t0 * R;
    for (int idx = tid; idx < ntok * R; idx += kBlock) {
        const int q = idx / R, r = idx - q * R;
        itr_tile[idx] = (uint8_t)((tokmask[q] >> r) & 1ull);
    }
    for (int r = tid; r < R; r += kBlock) {
        int n = 0;
        for (int q = 0; q < ntok; ++q) n += (int)((tokmask[q] >> r) & 1ull);
        tile_tpr[(size_t)j * R + r] = n;
    }
}

__global__ void __launch_bounds__(kBlock)
layout_scan_kernel(int E, int R, int align, Geometry geo, int32_t* __restrict__ tokens_per_expert,
                   int32_t* __restrict__ counts, int32_t* __restrict__ splits,
                   int32_t* __restrict__ tokens_per_rank, int32_t* __restrict__ offsets,
                   char* __restrict__ ws, WsLayout wl) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    int* sm = reinterpret_cast<int*>(smem_raw);
    __shared__ int scratch[kWarps + 1];
    __shared__ int am_last;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int El = E / R;
    int32_t* tile_base = reinterpret_cast<int32_t*>(ws + wl.tile_base);
    const int32_t* tile_tpr = reinterpret_cast<const int32_t*>(ws + wl.tile_tpr);
    int32_t* expert_count = reinterpret_cast<int32_t*>(ws + wl.expert_count);
    LayoutHeader* hdr = reinterpret_cast<LayoutHeader*>(ws);

    // ---- per-expert scan over tiles: one warp per expert ----
    int* bstart = sm + warp * (R + 1);  // exclusive prefix at each block start
    const int e = blockIdx.x * kWarps + warp;
    if (e < E) {
        for (int q = lane; q <= R; q += 32) bstart[q] = 0;
        __syncwarp();
        int32_t* rowp = tile_base + (size_t)e * geo.n_tiles;
        int running = 0;
        for (int c0 = 0; c0 < geo.n_tiles; c0 += 32) {
            const int jj = c0 + lane;
            const int v = (jj < geo.n_tiles) ? rowp[jj] : 0;
            int incl = v;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int n = __shfl_up_sync(kFull, incl, d);
                if (lane >= d) incl += n;
            }
            const int excl = running + incl - v;
            if (jj < geo.n_tiles) {
                rowp[jj] = excl;
                if (jj % geo.tpb == 0) bstart[jj / geo.tpb] = excl;
            }
            running += __shfl_sync(kFull, incl, 31);
        }
        __syncwarp();
        if (lane == 0) bstart[R] = running;
        __syncwarp();
        const int r = e / El, el = e - r * El;
        for (int sb = lane; sb < R; sb += 32)
            counts[((size_t)sb * R + r) * El + el] = bstart[sb + 1] - bstart[sb];
        if (lane == 0) {
            tokens_per_expert[e] = running;
            expert_count[e] = running;
        }
    }

    // ---- the last CTA to arrive finishes the cross-expert parts ----
    __threadfence();
    __syncthreads();
    if (tid == 0) am_last = (atomicAdd(&hdr->done, 1u) == gridDim.x - 1);
    __syncthreads();
    if (!am_last) return;
    __threadfence();

    int* padded = sm;  // reuse: [E]
    for (int q = tid; q < E; q += kBlock) {
        const int c = __ldcg(expert_count + q);
        padded[q] = ((c + align - 1) / align) * align;
    }
    __syncthreads();
    const int total = block_exclusive_scan<MOE_MAX_E / kBlock>(padded, E, scratch);
    for (int q = tid; q < E; q += kBlock) offsets[q] = padded[q];
    if (tid == 0) offsets[E] = total;

    for (int idx = tid; idx < R * R; idx += kBlock) {
        const int sb = idx / R, r = idx - sb * R;
        const int32_t* row = counts + ((size_t)sb * R + r) * El;
        int sum = 0;
        for (int el = 0; el < El; ++el) sum += __ldcg(row + el);
        splits[idx] = sum;
        int ntok = 0;
        for (int q = 0; q < geo.tpb; ++q) ntok += tile_tpr[(size_t)(sb * geo.tpb + q) * R + r];
        tokens_per_rank[idx] = ntok;
    }
    if (tid == 0) hdr->done = 0u;
}

cudaError_t launch_layout(const int64_t* topk_idx, int T, int K, int E, int R, int align,
                          int32_t* tokens_per_expert, int32_t* counts, int32_t* splits,
                          int32_t* tokens_per_rank, uint8_t* is_token_in_rank,
                          int32_t* expert_offsets, void* workspace, int32_t* status,
                          cudaStream_t stream) {
    const Geometry geo = layout_geometry(T, K, R);
    const WsLayout wl = workspace_layout(E, R, geo.n_tiles);
    char* ws = static_cast<char*>(workspace);

    const size_t hist_smem = sizeof(unsigned long long) * geo.TT + sizeof(int) * E;
    const int hist_grid = geo.n_tiles > 0 ? geo.n_tiles : 1;
    layout_hist_kernel<<<hist_grid, kBlock, hist_smem, stream>>>(topk_idx, T, K, E, R, geo,
                                                                 is_token_in_rank, ws, wl, status);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;

    const int scan_grid = (E + kWarps - 1) / kWarps;
    size_t scan_smem = sizeof(int) * (size_t)kWarps * (R + 1);
    if (scan_smem < sizeof(int) * (size_t)E) scan_smem = sizeof(int) * (size_t)E;
    layout_scan_kernel<<<scan_grid, kBlock, scan_smem, stream>>>(
        E, R, align, geo, tokens_per_expert, counts, splits, tokens_per_rank, expert_offsets, ws,
        wl);
    return cudaGetLastError();
}

}  // namespace moe
