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
//                       the permute) and its per-source-block counts; one warp
//                       per destination rank does the same for the per-tile
//                       distinct-token counts (tokens_per_rank); the last CTA
//                       to arrive then builds the padded offsets and splits
//                       from the other CTAs' results (arrival counter, no
//                       waiting).
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
    int* eidx = reinterpret_cast<int*>(tokmask + geo.TT);                          // [TT*K]
    uint16_t* crank = reinterpret_cast<uint16_t*>(eidx + geo.TT * K);               // [TT*K]
    uint16_t* cnt = crank + ((geo.TT * K + 1) & ~1);                                // [chunks][E]

    const int j = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (j == 0 && tid == 0) {
        LayoutHeader* h = reinterpret_cast<LayoutHeader*>(ws);
        h->off_tile_base = (int64_t)wl.tile_base;
        h->off_tile_tpr = (int64_t)wl.tile_tpr;
        h->off_expert_count = (int64_t)wl.expert_count;
        h->off_in_rank = (int64_t)wl.in_rank;
        h->magic = kLayoutMagic;
        h->T = T; h->K = K; h->E = E; h->R = R;
        h->TT = geo.TT; h->tpb = geo.tpb; h->n_tiles = geo.n_tiles;
        h->done = 0u;
    }
    if (j >= geo.n_tiles) return;

    int32_t* tile_base = reinterpret_cast<int32_t*>(ws + wl.tile_base);
    int32_t* tile_tpr = reinterpret_cast<int32_t*>(ws + wl.tile_tpr);
    uint16_t* in_rank = reinterpret_cast<uint16_t*>(ws + wl.in_rank);
    const int Tb = T / R, El = E / R;
    const int s = j / geo.tpb, i = j - s * geo.tpb;
    const int t0 = s * Tb + i * geo.TT;
    const int t1 = min(t0 + geo.TT, (s + 1) * Tb);
    const int ntok = t1 - t0, na = ntok * K;
    const int nchunks = (na + 31) / 32;

    for (int q = tid; q < nchunks * E; q += kBlock) cnt[q] = 0;
    for (int q = tid; q < ntok; q += kBlock) tokmask[q] = 0ull;
    __syncthreads();

    // Every warp ranks whole 32-assignment chunks of the tile (flat order):
    // lanes sharing an expert find each other with __match_any_sync; a
    // lane's rank inside its chunk is the number of lower lanes of the same
    // expert, and the chunk's count per expert is written by its leader.
    int bad = 0;
    const unsigned lt = lanemask_lt();
    for (int c = warp; c < nchunks; c += kWarps) {
        const int a = c * 32 + lane;
        int key = -1 - lane;
        if (a < na) {
            const int64_t e = topk[(int64_t)t0 * K + a];
            if (e >= 0 && e < E) key = (int)e; else bad = MOE_ST_EXPERT_OOR;
            eidx[a] = key >= 0 ? key : -1;
        }
        const unsigned peers = __match_any_sync(kFull, key);
        if (key >= 0) {
            crank[a] = (uint16_t)__popc(peers & lt);
            if (lane == __ffs(peers) - 1) cnt[c * E + key] = (uint16_t)__popc(peers);
            atomicOr(&tokmask[a / K], 1ull << (key / El));
        }
    }
    warp_status_or(status, bad);
    __syncthreads();

    // In-tile stable rank = assignments of the same expert in earlier chunks
    // + rank inside the chunk.
    uint16_t* out_rank = in_rank + (size_t)t0 * K;
    for (int a = tid; a < na; a += kBlock) {
        const int e = eidx[a];
        if (e < 0) { out_rank[a] = 0xFFFFu; continue; }
        int before = 0;
        for (int c = 0; c < a / 32; ++c) before += cnt[c * E + e];
        out_rank[a] = (uint16_t)(before + crank[a]);
    }
    for (int e = tid; e < E; e += kBlock) {
        int total = 0;
        for (int c = 0; c < nchunks; ++c) total += cnt[c * E + e];
        tile_base[(size_t)e * geo.n_tiles + j] = total;
    }
    uint8_t* itr_tile = itr + (size_t)t0 * R;
    for (int idx = tid; idx < ntok * R; idx += kBlock) {
        const int q = idx / R, r = idx - q * R;
        itr_tile[idx] = (uint8_t)((tokmask[q] >> r) & 1ull);
    }
    for (int r = tid; r < R; r += kBlock) {
        int n = 0;
        for (int q = 0; q < ntok; ++q) n += (int)((tokmask[q] >> r) & 1ull);
        tile_tpr[(size_t)r * geo.n_tiles + j] = n;     // rank-major, like tile_base
    }
}

constexpr int kScanBatch = 32;  // 32-tile chunks loaded per batch (independent loads)

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
    const int n_tiles = geo.n_tiles;
    int32_t* tile_base = reinterpret_cast<int32_t*>(ws + wl.tile_base);
    int32_t* tile_tpr = reinterpret_cast<int32_t*>(ws + wl.tile_tpr);
    int32_t* expert_count = reinterpret_cast<int32_t*>(ws + wl.expert_count);
    LayoutHeader* hdr = reinterpret_cast<LayoutHeader*>(ws);

    // ---- one warp per row of per-tile counts: rows 0..E-1 are experts, rows
    // E..E+R-1 are destination ranks (distinct tokens per tile).  Each warp
    // computes the exclusive scan of its row over the tiles (written back in
    // place for experts: the stable per-tile bases the permute reads) and the
    // sum over each source block's tiles.  Loads come in batches of
    // kScanBatch coalesced 32-tile chunks, all issued before they are used.
    int* bstart = sm + warp * (R + 1);
    const int p = blockIdx.x * kWarps + warp;
    if (p < E + R) {
        const bool is_expert = p < E;
        int32_t* rowp = is_expert ? tile_base + (size_t)p * n_tiles
                                  : tile_tpr + (size_t)(p - E) * n_tiles;
        for (int q = lane; q <= R; q += 32) bstart[q] = 0;
        __syncwarp();
        int running = 0;
        for (int c0 = 0; c0 < n_tiles; c0 += 32 * kScanBatch) {
            int v[kScanBatch];
#pragma unroll
            for (int b = 0; b < kScanBatch; ++b) {
                const int jj = c0 + b * 32 + lane;
                v[b] = (jj < n_tiles) ? rowp[jj] : 0;
            }
#pragma unroll
            for (int b = 0; b < kScanBatch; ++b) {
                int incl = v[b];
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const int n = __shfl_up_sync(kFull, incl, d);
                    if (lane >= d) incl += n;
                }
                const int jj = c0 + b * 32 + lane;
                const int excl = running + incl - v[b];
                if (jj < n_tiles) {
                    if (is_expert) rowp[jj] = excl;
                    if (jj % geo.tpb == 0) bstart[jj / geo.tpb] = excl;
                }
                running += __shfl_sync(kFull, incl, 31);
            }
        }
        __syncwarp();
        if (lane == 0) bstart[R] = running;
        __syncwarp();
        if (is_expert) {
            const int r = p / El, el = p - r * El;
            for (int sb = lane; sb < R; sb += 32)
                counts[((size_t)sb * R + r) * El + el] = bstart[sb + 1] - bstart[sb];
            if (lane == 0) {
                tokens_per_expert[p] = running;
                expert_count[p] = running;
            }
        } else {
            const int r = p - E;
            for (int sb = lane; sb < R; sb += 32)
                tokens_per_rank[(size_t)sb * R + r] = bstart[sb + 1] - bstart[sb];
        }
    }

    // ---- the last CTA to arrive finishes the cross-expert parts ----
    __threadfence();
    __syncthreads();
    if (tid == 0) am_last = (atomicAdd(&hdr->done, 1u) == gridDim.x - 1);
    __syncthreads();
    if (!am_last) return;
    __threadfence();

    int* padded = sm;            // [E]
    int* acc_splits = sm + E;    // [R*R]
    for (int q = tid; q < E; q += kBlock) {
        const int c = __ldcg(expert_count + q);
        padded[q] = ((c + align - 1) / align) * align;
    }
    for (int q = tid; q < R * R; q += kBlock) acc_splits[q] = 0;
    __syncthreads();
    const int total = block_exclusive_scan<MOE_MAX_E / kBlock>(padded, E, scratch);
    for (int q = tid; q < E; q += kBlock) offsets[q] = padded[q];
    if (tid == 0) offsets[E] = total;

    // splits[s][r] = sum over el of counts[s][r][el]; counts is [R*R][El]
    // contiguous: load a batch of elements per thread (coalesced), then add
    // each to its (s, r) bin in shared memory.
    const int n = R * E;
    constexpr int kSplitBatch = 8;
    for (int base = 0; base < n; base += kBlock * kSplitBatch) {
        int v[kSplitBatch];
#pragma unroll
        for (int b = 0; b < kSplitBatch; ++b) {
            const int i = base + b * kBlock + tid;
            v[b] = (i < n) ? __ldcg(counts + i) : 0;
        }
#pragma unroll
        for (int b = 0; b < kSplitBatch; ++b) {
            const int i = base + b * kBlock + tid;
            if (i < n && v[b]) atomicAdd(&acc_splits[i / El], v[b]);
        }
    }
    __syncthreads();
    for (int q = tid; q < R * R; q += kBlock) splits[q] = acc_splits[q];
    if (tid == 0) hdr->done = 0u;
}

cudaError_t launch_layout(const int64_t* topk_idx, int T, int K, int E, int R, int align,
                          int32_t* tokens_per_expert, int32_t* counts, int32_t* splits,
                          int32_t* tokens_per_rank, uint8_t* is_token_in_rank,
                          int32_t* expert_offsets, void* workspace, int32_t* status,
                          cudaStream_t stream) {
    const Geometry geo = layout_geometry(T, K, R);
    const WsLayout wl = workspace_layout(E, R, geo.n_tiles, (int64_t)T * K);
    char* ws = static_cast<char*>(workspace);

    const int na_max = geo.TT * K;
    const size_t hist_smem = sizeof(unsigned long long) * geo.TT + sizeof(int) * na_max +
                             sizeof(uint16_t) * ((na_max + 1) & ~1) +
                             sizeof(uint16_t) * (size_t)((na_max + 31) / 32) * E;
    const int hist_grid = geo.n_tiles > 0 ? geo.n_tiles : 1;
    layout_hist_kernel<<<hist_grid, kBlock, hist_smem, stream>>>(topk_idx, T, K, E, R, geo,
                                                                 is_token_in_rank, ws, wl, status);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;

    const int scan_grid = (E + R + kWarps - 1) / kWarps;
    size_t scan_smem = sizeof(int) * (size_t)kWarps * (R + 1);
    const size_t last_smem = sizeof(int) * ((size_t)E + (size_t)R * R);
    if (scan_smem < last_smem) scan_smem = last_smem;
    layout_scan_kernel<<<scan_grid, kBlock, scan_smem, stream>>>(
        E, R, align, geo, tokens_per_expert, counts, splits, tokens_per_rank, expert_offsets, ws,
        wl);
    return cudaGetLastError();
}

}  // namespace moe
