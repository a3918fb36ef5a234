// layout.cu -- routing layout on the device (get_dispatch_layout of the DeepEP
// issue "Does Deepep's Dispatch/Combine Support Autograd Like PyTorch's
// all_to_all?"; the count matrix [ep_size, E_local] of the DeepSpeed PR
// "Derive AutoEP rank splits from the per-expert count exchange", Redundancy;
// the group alignment of the DeepSpeed AutoEP base PR, Attribution).
//
// Two short kernels in stream order, chained with programmatic dependent
// launch: no host synchronisation, no grid barrier, no cooperative launch and
// nothing to zero before the call.  Tiles of <= TT consecutive tokens (at
// least 512 assignments each and at most about one per SM, never straddling
// a source rank's token block):
//   layout_tiles_kernel: one 1024-thread CTA per tile ranks its assignments
//     (in-tile stable ranks, per-tile count of every expert, distinct tokens
//     per destination rank, is_token_in_rank);
//   layout_rows_kernel: one warp per row of per-tile counts scans it over the
//     tiles (the per-tile bases the permute reads), sums it per source block
//     (count matrix, tokens_per_rank, splits) and totals it
//     (tokens_per_expert); the last CTA to finish computes the offsets.
// Each kernel waits for its predecessor's grid (griddepcontrol.wait) before
// reading its output and lets its successor be scheduled at once, so the
// launches overlap and the permute that follows starts as soon as the
// offsets are written.
//
// Bytes: reads topk_idx once (8*A), writes the [T,R] flags, in-tile ranks
// (2*A) and O((E+R) * tiles) ints.
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kLThreads = 1024;                  // tile kernel: one CTA per tile
constexpr int kLWarps = kLThreads / 32;
constexpr int kRowWarps = kWarps;                // row kernel: one warp per row
constexpr int kRowWarpsOne = 32;                 // ... or one CTA for at most 32 rows
constexpr int kRowBatch = 8;                     // row values loaded per lane at a time

// ------------------------------------------------------------- tiles ---
//
// One 1024-thread CTA per tile j (tokens [t0, t1) of source block s): each
// warp ranks whole 32-assignment chunks in flat order with __match_any_sync
// (lanes sharing an expert find each other; a lane's rank is the number of
// lower lanes of its expert), recording the chunk's count per expert; a
// per-expert exclusive scan of the chunk counts gives every assignment's
// stable in-tile rank and the tile's count of the expert (tile_base[e][j]);
// token masks of destination ranks give is_token_in_rank and the tile's
// distinct tokens per rank (tile_tpr[r][j]).  CTA 0 also writes the header and
// zeroes what the row kernel accumulates into (its arrival counter and the
// splits), which the row kernel reads only after this grid has completed.
__global__ void __launch_bounds__(kLThreads, 1)
layout_tiles_kernel(const int64_t* __restrict__ topk, int T, int K, int E, int R, Geometry geo,
                    int32_t* __restrict__ splits, uint8_t* __restrict__ itr,
                    char* __restrict__ ws, WsLayout wl, int32_t* __restrict__ status) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int j = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int Tb = T / R, El = E / R;
    const int n_tiles = geo.n_tiles;
    int32_t* tile_base = reinterpret_cast<int32_t*>(ws + wl.tile_base);
    int32_t* tile_tpr = reinterpret_cast<int32_t*>(ws + wl.tile_tpr);
    uint16_t* in_rank = reinterpret_cast<uint16_t*>(ws + wl.in_rank);
    LayoutHeader* hdr = reinterpret_cast<LayoutHeader*>(ws);
    pdl_wait();        // topk_idx may be the previous kernel's output
    pdl_trigger();

    if (j == 0) {
        if (tid == 0) {
            hdr->off_tile_base = (int64_t)wl.tile_base;
            hdr->off_tile_tpr = (int64_t)wl.tile_tpr;
            hdr->off_expert_count = (int64_t)wl.expert_count;
            hdr->off_in_rank = (int64_t)wl.in_rank;
            hdr->magic = kLayoutMagic;
            hdr->T = T; hdr->K = K; hdr->E = E; hdr->R = R;
            hdr->TT = geo.TT; hdr->tpb = geo.tpb; hdr->n_tiles = n_tiles;
            hdr->done = 0u;
        }
        for (int q = tid; q < R * R; q += kLThreads) splits[q] = 0;
    }
    if (j >= n_tiles) return;

    unsigned long long* tokmask = reinterpret_cast<unsigned long long*>(smem_raw);  // [TT]
    int* eidx = reinterpret_cast<int*>(tokmask + geo.TT);                          // [TT*K]
    uint16_t* crank = reinterpret_cast<uint16_t*>(eidx + geo.TT * K);               // [TT*K]
    uint16_t* cnt = crank + ((geo.TT * K + 1) & ~1);                                // [chunks][E]
    const int s = j / geo.tpb, i = j - s * geo.tpb;
    const int t0 = s * Tb + i * geo.TT;
    const int t1 = min(t0 + geo.TT, (s + 1) * Tb);
    const int ntok = t1 - t0, na = ntok * K;
    const int nchunks = (na + 31) / 32;

    for (int q = tid; q < nchunks * E; q += kLThreads) cnt[q] = 0;
    for (int q = tid; q < ntok; q += kLThreads) tokmask[q] = 0ull;
    __syncthreads();

    int bad = 0;
    const unsigned lt = lanemask_lt();
    for (int c = warp; c < nchunks; c += kLWarps) {      // warp-uniform
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

    // Per expert, an exclusive scan of the chunk counts over the chunks (in
    // place); its total is the tile's count of the expert.
    for (int e = tid; e < E; e += kLThreads) {
        int run = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int v = cnt[c * E + e];
            cnt[c * E + e] = (uint16_t)run;
            run += v;
        }
        tile_base[(size_t)e * n_tiles + j] = run;
    }
    __syncthreads();
    uint16_t* out_rank = in_rank + (size_t)t0 * K;
    for (int a = tid; a < na; a += kLThreads) {
        const int e = eidx[a];
        out_rank[a] = e < 0 ? (uint16_t)0xFFFFu : (uint16_t)(cnt[(a >> 5) * E + e] + crank[a]);
    }
    uint8_t* itr_tile = itr + (size_t)t0 * R;
    for (int idx = tid; idx < ntok * R; idx += kLThreads) {
        const int q = idx / R, r = idx - q * R;
        itr_tile[idx] = (uint8_t)((tokmask[q] >> r) & 1ull);
    }
    // Distinct tokens of the tile per destination rank: a warp per rank.
    for (int r = warp; r < R; r += kLWarps) {
        int n = 0;
        for (int q = lane; q < ntok; q += 32) n += (int)((tokmask[q] >> r) & 1ull);
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) n += __shfl_xor_sync(kFull, n, d);
        if (lane == 0) tile_tpr[(size_t)r * n_tiles + j] = n;   // rank-major, like tile_base
    }
}

// -------------------------------------------------------------- rows ---
//
// One warp per row p of per-tile counts -- expert rows p < E, then one row
// per destination rank: each lane loads its contiguous segment of the row
// (kRowBatch independent loads at a time), the warp scans the segment sums,
// and each lane rewrites its segment as exclusive prefixes (expert rows:
// the per-tile stable bases the permute reads), noting the prefix at the
// first tile of every source block.  Block differences give the count matrix
// (expert rows; summed per destination rank into the splits) or
// tokens_per_rank (rank rows); an expert row's total is tokens_per_expert
// and the per-expert count the permute reads.  The last CTA to finish (an
// arrival counter the tile kernel zeroed; no CTA waits) turns the totals
// into the padded exclusive offsets.  With ONE (E + R <= 32: one CTA of 32
// warps holds every row) there is no last CTA to find: after one barrier,
// warp 0 scans the padded totals the row warps left in shared memory: no
// fence, no arrival atomic, no re-read of the totals (measured on the
// Mixtral shape: eager layout 13.3 -> 11.4 us; in a graph, where the next
// kernel's launch overlaps, the dispatch segment 28.9 -> 28.8 us).
template <int RW, bool ONE>
__global__ void __launch_bounds__(RW * 32)
layout_rows_kernel(int E, int R, int align, Geometry geo, int32_t* __restrict__ tokens_per_expert,
                   int32_t* __restrict__ counts, int32_t* __restrict__ splits,
                   int32_t* __restrict__ tokens_per_rank, int32_t* __restrict__ offsets,
                   char* __restrict__ ws, WsLayout wl) {
    static_assert(!ONE || RW == 32, "one CTA: a warp per row, 32 rows at most");
    __shared__ int bs_all[RW][MOE_MAX_R + 1];
    __shared__ int ctot[MOE_MAX_E + 1];
    __shared__ int scratch[kWarps + 1];
    __shared__ int am_last;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n_tiles = geo.n_tiles, tpb = geo.tpb, El = E / R;
    int32_t* tile_base = reinterpret_cast<int32_t*>(ws + wl.tile_base);
    int32_t* tile_tpr = reinterpret_cast<int32_t*>(ws + wl.tile_tpr);
    int32_t* expert_count = reinterpret_cast<int32_t*>(ws + wl.expert_count);
    LayoutHeader* hdr = reinterpret_cast<LayoutHeader*>(ws);
    pdl_wait();
    pdl_trigger();

    const int p = blockIdx.x * RW + warp;                  // warp-uniform
    if (p < E + R) {
        const bool is_expert = p < E;
        int32_t* row = is_expert ? tile_base + (size_t)p * n_tiles
                                 : tile_tpr + (size_t)(p - E) * n_tiles;
        int* bs = bs_all[warp];
        for (int q = lane; q <= R; q += 32) bs[q] = 0;
        __syncwarp();
        const int seg = (n_tiles + 31) / 32;
        const int j0 = min(lane * seg, n_tiles), j1 = min(j0 + seg, n_tiles);
        // The first batch stays in registers for the second pass (rows of
        // up to 32 * kRowBatch tiles are read once).
        int first[kRowBatch];
        int local = 0;
#pragma unroll
        for (int q = 0; q < kRowBatch; ++q) {
            first[q] = (j0 + q < j1) ? __ldcg(row + j0 + q) : 0;
            local += first[q];
        }
        for (int b = j0 + kRowBatch; b < j1; b += kRowBatch) {
            int v[kRowBatch];
#pragma unroll
            for (int q = 0; q < kRowBatch; ++q) v[q] = (b + q < j1) ? __ldcg(row + b + q) : 0;
#pragma unroll
            for (int q = 0; q < kRowBatch; ++q) local += v[q];
        }
        int incl = local;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int x = __shfl_up_sync(kFull, incl, d);
            if (lane >= d) incl += x;
        }
        const int total = __shfl_sync(kFull, incl, 31);
        int run = incl - local;
        // First tile of a source block at or after j0 (tiles of block sb are
        // [sb*tpb, (sb+1)*tpb)); tpb >= 1 whenever a lane holds a tile.
        int nb = j0 < j1 ? (j0 + tpb - 1) / tpb * tpb : 0;
        for (int b = j0; b < j1; b += kRowBatch) {
            int v[kRowBatch];
            if (b == j0) {
#pragma unroll
                for (int q = 0; q < kRowBatch; ++q) v[q] = first[q];
            } else {
#pragma unroll
                for (int q = 0; q < kRowBatch; ++q) v[q] = (b + q < j1) ? __ldcg(row + b + q) : 0;
            }
#pragma unroll
            for (int q = 0; q < kRowBatch; ++q) {
                const int jj = b + q;
                if (jj < j1) {
                    if (is_expert) row[jj] = run;
                    if (jj == nb) {
                        bs[jj / tpb] = run;
                        nb += tpb;
                    }
                    run += v[q];
                }
            }
        }
        __syncwarp();
        if (lane == 0) bs[R] = total;
        __syncwarp();
        if (is_expert) {
            const int r = p / El, el = p - r * El;
            for (int sb = lane; sb < R; sb += 32) {
                const int c = bs[sb + 1] - bs[sb];
                counts[((size_t)sb * R + r) * El + el] = c;
                if (c) atomicAdd(&splits[sb * R + r], c);
            }
            if (lane == 0) {
                tokens_per_expert[p] = total;
                expert_count[p] = total;
                if (ONE) ctot[p] = ((total + align - 1) / align) * align;
            }
        } else {
            const int r = p - E;
            for (int sb = lane; sb < R; sb += 32)
                tokens_per_rank[(size_t)sb * R + r] = bs[sb + 1] - bs[sb];
        }
    }

    if constexpr (ONE) {
        // Every row is this CTA's: the padded totals are in shared memory.
        __syncthreads();
        if (warp == 0) {
            const int c = lane < E ? ctot[lane] : 0;    // E <= 31
            int incl = c;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int x = __shfl_up_sync(kFull, incl, d);
                if (lane >= d) incl += x;
            }
            if (lane < E) offsets[lane] = incl - c;
            if (lane == E - 1) offsets[E] = incl;
        }
        return;
    }
    // The last CTA to finish computes the offsets from every expert's total.
    __threadfence();
    __syncthreads();
    if (tid == 0) am_last = (atomicAdd(&hdr->done, 1u) == gridDim.x - 1);
    __syncthreads();
    if (!am_last) return;
    __threadfence();
    for (int e = tid; e < E; e += kBlock) {
        const int c = __ldcg(expert_count + e);
        ctot[e] = ((c + align - 1) / align) * align;
    }
    __syncthreads();
    const int total = block_exclusive_scan<MOE_MAX_E / kBlock>(ctot, E, scratch);
    for (int e = tid; e < E; e += kBlock) offsets[e] = ctot[e];
    if (tid == 0) offsets[E] = total;
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
    const size_t smem = sizeof(unsigned long long) * geo.TT + sizeof(int) * na_max +
                        sizeof(uint16_t) * ((na_max + 1) & ~1) +
                        sizeof(uint16_t) * (size_t)((na_max + 31) / 32) * E;
    // Per-device cache of the shared-memory opt-in (host threads may call
    // concurrently: atomics).
    static std::atomic<int> configured[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    if (smem > 48 * 1024 &&
        (dev < 0 || dev >= 64 || configured[dev].load(std::memory_order_relaxed) < (int)smem)) {
        const cudaError_t e = cudaFuncSetAttribute(
            layout_tiles_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) {
            int cur = configured[dev].load(std::memory_order_relaxed);
            while (cur < (int)smem &&
                   !configured[dev].compare_exchange_weak(cur, (int)smem, std::memory_order_relaxed)) {
            }
        }
    }
    const int grid = geo.n_tiles > 0 ? geo.n_tiles : 1;
    cudaError_t err = launch_pdl(layout_tiles_kernel, dim3(grid), dim3(kLThreads), smem, stream,
                                 topk_idx, T, K, E, R, geo, splits, is_token_in_rank, ws, wl,
                                 status);
    if (err != cudaSuccess) return err;
#ifndef MOE_LAYOUT_ONE
#define MOE_LAYOUT_ONE 1
#endif
    if (MOE_LAYOUT_ONE && E + R <= kRowWarpsOne)
        return launch_pdl(layout_rows_kernel<kRowWarpsOne, true>, dim3(1), dim3(kRowWarpsOne * 32),
                          0, stream, E, R, align, geo, tokens_per_expert, counts, splits,
                          tokens_per_rank, expert_offsets, ws, wl);
    const int rows_grid = (E + R + kRowWarps - 1) / kRowWarps;
    return launch_pdl(layout_rows_kernel<kRowWarps, false>, dim3(rows_grid), dim3(kBlock), 0, stream, E, R, align,
                      geo, tokens_per_expert, counts, splits, tokens_per_rank, expert_offsets, ws,
                      wl);
}

}  // namespace moe
