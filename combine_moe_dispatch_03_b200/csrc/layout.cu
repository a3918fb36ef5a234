// layout.cu -- routing layout on the device (get_dispatch_layout of the DeepEP
// issue "Does Deepep's Dispatch/Combine Support Autograd Like PyTorch's
// all_to_all?"; the count matrix [ep_size, E_local] of the DeepSpeed PR
// "Derive AutoEP rank splits from the per-expert count exchange", Redundancy;
// the group alignment of the DeepSpeed AutoEP base PR, Attribution).
//
// One kernel, no host synchronisation.  Tiles of <= TT consecutive tokens
// (at most 148, never straddling a source rank's token block) each get a
// 1024-thread CTA:
//   phase 1 (every CTA, its tile): each warp ranks whole 32-assignment chunks
//     in flat order with __match_any_sync (lanes sharing an expert find each
//     other; a lane's rank is the number of lower lanes of its expert); the
//     chunk counts give every assignment's stable in-tile rank and the tile's
//     per-expert count; token rank masks give is_token_in_rank and the tile's
//     distinct tokens per destination rank.
//   phase 2: one warp per row of per-tile counts -- experts, then destination
//     ranks -- scans the row over the tiles (the expert rows are rewritten in
//     place as the per-tile stable bases the permute reads) and sums it per
//     source block (count matrix, tokens_per_rank).
//   phase 3: padded exclusive offsets and splits.
// When every tile's CTA fits on the GPU at once the launch is cooperative:
// phase 1 also adds each tile's per-expert counts and per-destination-rank
// sums into zeroed accumulators in the workspace (atomics), so one grid
// barrier (a bounded spin on a counter that records MOE_ST_TIMEOUT instead
// of hanging) separates phase 1 from everything else: after it, CTA 0 runs
// phase 3 from the accumulated totals while the warps of the other CTAs scan
// the rows, each lane holding its segment of a row in registers.  Otherwise
// the last CTA to arrive (an arrival counter, no waiting) runs phases 2 and 3
// alone.  The counter and the accumulators sit at the start of the workspace
// and are zeroed by one memset enqueued just before the kernel.
//
// Bytes: reads topk_idx once (8*A), writes the [T,R] flags, in-tile ranks
// (2*A) and O((E+R) * tiles) ints.
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kLThreads = 1024;
constexpr int kLWarps = kLThreads / 32;
constexpr size_t kLayoutSmemMax = 200 * 1024;   // staging limit for phase 2

// In-place exclusive scan of n <= kLThreads ints in shared memory by a
// 1024-thread CTA; returns the total.  `scratch` holds kLWarps + 1 ints.
__device__ int block_exclusive_scan_1024(int* data, int n, int* scratch) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int v = tid < n ? data[tid] : 0;
    int incl = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int x = __shfl_up_sync(kFull, incl, d);
        if (lane >= d) incl += x;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = scratch[lane];
        int wi = w;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int x = __shfl_up_sync(kFull, wi, d);
            if (lane >= d) wi += x;
        }
        scratch[lane] = wi - w;
        if (lane == 31) scratch[kLWarps] = wi;
    }
    __syncthreads();
    if (tid < n) data[tid] = scratch[warp] + incl - v;
    const int total = scratch[kLWarps];
    __syncthreads();
    return total;
}

constexpr uint64_t kBarrierLimitNs = 2000000000ull;   // 2 s

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Grid barrier for a cooperative launch: every CTA adds one arrival to
// `bar` (zeroed before the launch) and waits until `target` arrivals.  The
// wait is bounded by limit_ns of %globaltimer; returns false if it gave up.
__device__ bool grid_barrier(unsigned* bar, unsigned target, uint64_t limit_ns) {
    __shared__ int ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(bar, 1u);
        const uint64_t t0 = global_timer_ns();
        int good = 1;
        for (;;) {
            unsigned v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
            if (v >= target) break;
            if (global_timer_ns() - t0 > limit_ns) { good = 0; break; }
            __nanosleep(64);
        }
        __threadfence();
        ok = good;
    }
    __syncthreads();
    return ok != 0;
}

// Phase 2 for one row p of per-tile counts (all 32 lanes): exclusive scan
// over the tiles with lane-contiguous segments, written back in place for
// expert rows; block sums into the count matrix / tokens_per_rank.  `rows`
// is the row in shared memory when staged, else nullptr (global).
struct RowOut {
    int total;
};
__device__ RowOut scan_row(int p, int E, int R, const Geometry& geo, int32_t* tile_base,
                           int32_t* tile_tpr, int* smem_row, int* bs, int32_t* counts,
                           int32_t* tokens_per_rank) {
    const int lane = threadIdx.x & 31;
    const int n_tiles = geo.n_tiles, El = E / R;
    const bool is_expert = p < E;
    int32_t* rowg = is_expert ? tile_base + (size_t)p * n_tiles
                              : tile_tpr + (size_t)(p - E) * n_tiles;
    int* rows = smem_row ? smem_row : rowg;
    for (int q = lane; q <= R; q += 32) bs[q] = 0;
    __syncwarp();
    const int seg = (n_tiles + 31) / 32;
    const int j0 = min(lane * seg, n_tiles), j1 = min(j0 + seg, n_tiles);
    int local = 0;
    for (int jj = j0; jj < j1; ++jj) local += smem_row ? rows[jj] : __ldcg(rowg + jj);
    int incl = local;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int x = __shfl_up_sync(kFull, incl, d);
        if (lane >= d) incl += x;
    }
    const int total = __shfl_sync(kFull, incl, 31);
    int run = incl - local;
    // Source block of tile jj (tiles of block sb are [sb*tpb, (sb+1)*tpb)),
    // tracked incrementally instead of divided out per tile.
    int nb = j0 < j1 ? (j0 + geo.tpb - 1) / geo.tpb * geo.tpb : 0;   // first block start >= j0
    for (int jj = j0; jj < j1; ++jj) {
        const int v = smem_row ? rows[jj] : __ldcg(rowg + jj);
        if (is_expert) rows[jj] = run;
        if (jj == nb) {
            bs[jj / geo.tpb] = run;
            nb += geo.tpb;
        }
        run += v;
    }
    __syncwarp();
    if (lane == 0) bs[R] = total;
    __syncwarp();
    if (is_expert) {
        const int r = p / El, el = p - r * El;
        for (int sb = lane; sb < R; sb += 32)
            counts[((size_t)sb * R + r) * El + el] = bs[sb + 1] - bs[sb];
    } else {
        const int r = p - E;
        for (int sb = lane; sb < R; sb += 32)
            tokens_per_rank[(size_t)sb * R + r] = bs[sb + 1] - bs[sb];
    }
    __syncwarp();
    RowOut o;
    o.total = total;
    return o;
}

// Phase 2 for one row p in the cooperative path, where the grid has at
// most kCoopMaxTiles tiles: each lane loads its segment of the row once into
// registers (independent loads, one L2 round trip), then the same exclusive
// scan and per-block sums as scan_row.
constexpr int kCoopSeg = 5;
constexpr int kCoopMaxTiles = 32 * kCoopSeg;

__device__ void scan_row_regs(int p, int E, int R, const Geometry& geo, int32_t* tile_base,
                              int32_t* tile_tpr, int* bs, int32_t* counts,
                              int32_t* tokens_per_rank) {
    const int lane = threadIdx.x & 31;
    const int n_tiles = geo.n_tiles, El = E / R;
    const bool is_expert = p < E;
    int32_t* rowg = is_expert ? tile_base + (size_t)p * n_tiles
                              : tile_tpr + (size_t)(p - E) * n_tiles;
    for (int q = lane; q <= R; q += 32) bs[q] = 0;
    __syncwarp();
    const int seg = (n_tiles + 31) / 32;
    const int j0 = min(lane * seg, n_tiles), j1 = min(j0 + seg, n_tiles);
    int v[kCoopSeg];
    int local = 0;
#pragma unroll
    for (int i = 0; i < kCoopSeg; ++i) {
        v[i] = (j0 + i < j1) ? __ldcg(rowg + j0 + i) : 0;
        local += v[i];
    }
    int incl = local;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int x = __shfl_up_sync(kFull, incl, d);
        if (lane >= d) incl += x;
    }
    const int total = __shfl_sync(kFull, incl, 31);
    int run = incl - local;
#pragma unroll
    for (int i = 0; i < kCoopSeg; ++i) {
        const int jj = j0 + i;
        if (jj < j1) {
            if (is_expert) rowg[jj] = run;
            if (jj % geo.tpb == 0) bs[jj / geo.tpb] = run;
            run += v[i];
        }
    }
    __syncwarp();
    if (lane == 0) bs[R] = total;
    __syncwarp();
    if (is_expert) {
        const int r = p / El, el = p - r * El;
        for (int sb = lane; sb < R; sb += 32)
            counts[((size_t)sb * R + r) * El + el] = bs[sb + 1] - bs[sb];
    } else {
        const int r = p - E;
        for (int sb = lane; sb < R; sb += 32)
            tokens_per_rank[(size_t)sb * R + r] = bs[sb + 1] - bs[sb];
    }
    __syncwarp();
}

// Phases 2 and 3 by one CTA (all kLThreads threads), after phase 1 has
// produced every tile's per-expert counts and per-rank distinct tokens:
// one warp per row scans it over the tiles (rewriting expert rows as the
// per-tile stable bases) and sums it per source block; the row totals give
// tokens_per_expert, the per-expert counts the permute reads and, padded and
// scanned, the offsets; the block sums of the expert rows give the splits.
// `mat` holds the rows [E+R][n_tiles] in shared memory when staged (copied
// back to tile_base at the end), else nullptr (rows read in global memory).
// `acc_splits` must be zeroed by the caller before a __syncthreads().
__device__ void phases_2_3_one_cta(int E, int R, int align, const Geometry& geo, int* mat,
                                   int* bstart, int* ctot, int* acc_splits, int* scratch,
                                   int32_t* tile_base, int32_t* tile_tpr, int32_t* expert_count,
                                   int32_t* tokens_per_expert, int32_t* counts, int32_t* splits,
                                   int32_t* tokens_per_rank, int32_t* offsets) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int El = E / R, n_tiles = geo.n_tiles, nrows = E + R;
    int* bs = bstart + warp * (R + 1);
    for (int p = warp; p < nrows; p += kLWarps) {
        const RowOut o = scan_row(p, E, R, geo, tile_base, tile_tpr,
                                  mat ? mat + (size_t)p * n_tiles : nullptr, bs, counts,
                                  tokens_per_rank);
        if (p < E) {
            const int r = p / El;
            for (int sb = lane; sb < R; sb += 32)
                atomicAdd(&acc_splits[sb * R + r], bs[sb + 1] - bs[sb]);
            if (lane == 0) {
                tokens_per_expert[p] = o.total;
                expert_count[p] = o.total;
                ctot[p] = o.total;
            }
        }
        __syncwarp();
    }
    __syncthreads();
    if (mat) {
        const int ne = E * n_tiles;
        for (int q = tid; q < ne; q += kLThreads) tile_base[q] = mat[q];
    }
    // phase 3: offsets and splits
    if (tid < E) ctot[tid] = ((ctot[tid] + align - 1) / align) * align;
    __syncthreads();
    const int total = block_exclusive_scan_1024(ctot, E, scratch);
    if (tid < E) offsets[tid] = ctot[tid];
    if (tid == 0) offsets[E] = total;
    for (int q = tid; q < R * R; q += kLThreads) splits[q] = acc_splits[q];
}

__global__ void __launch_bounds__(kLThreads, 1)
layout_kernel(const int64_t* __restrict__ topk, int T, int K, int E, int R, int align,
              Geometry geo, int32_t* __restrict__ tokens_per_expert, int32_t* __restrict__ counts,
              int32_t* __restrict__ splits, int32_t* __restrict__ tokens_per_rank,
              uint8_t* __restrict__ itr, int32_t* __restrict__ offsets, char* __restrict__ ws,
              WsLayout wl, int32_t* __restrict__ status, int coop, int staged,
              unsigned bar_extra, uint64_t bar_limit_ns) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ int scratch[kLWarps + 1];
    __shared__ int am_last;
    __shared__ int rank_sum[MOE_MAX_R];
    const int j = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int Tb = R > 0 ? T / R : 0, El = E / R;
    const int n_tiles = geo.n_tiles;
    int32_t* tile_base = reinterpret_cast<int32_t*>(ws + wl.tile_base);
    int32_t* tile_tpr = reinterpret_cast<int32_t*>(ws + wl.tile_tpr);
    int32_t* expert_count = reinterpret_cast<int32_t*>(ws + wl.expert_count);
    int32_t* splits_acc = reinterpret_cast<int32_t*>(ws + wl.splits_acc);
    uint16_t* in_rank = reinterpret_cast<uint16_t*>(ws + wl.in_rank);
    LayoutHeader* hdr = reinterpret_cast<LayoutHeader*>(ws);

    if (j == 0 && tid == 0) {
        hdr->off_tile_base = (int64_t)wl.tile_base;
        hdr->off_tile_tpr = (int64_t)wl.tile_tpr;
        hdr->off_expert_count = (int64_t)wl.expert_count;
        hdr->off_in_rank = (int64_t)wl.in_rank;
        hdr->magic = kLayoutMagic;
        hdr->T = T; hdr->K = K; hdr->E = E; hdr->R = R;
        hdr->TT = geo.TT; hdr->tpb = geo.tpb; hdr->n_tiles = n_tiles;
    }

    // ------------------------------------------------- phase 1: one tile ---
    if (j < n_tiles) {
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
        if (tid < R) rank_sum[tid] = 0;
        __syncthreads();

        int bad = 0;
        const unsigned lt = lanemask_lt();
        for (int c = warp; c < nchunks; c += kLWarps) {
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

        // Per expert, an exclusive scan of the chunk counts over the chunks
        // (in place); its total is the tile's count of the expert.  The
        // in-tile stable rank is then the scan at the assignment's chunk plus
        // its rank inside the chunk.
        for (int e = tid; e < E; e += kLThreads) {
            int run = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int v = cnt[c * E + e];
                cnt[c * E + e] = (uint16_t)run;
                run += v;
            }
            tile_base[(size_t)e * n_tiles + j] = run;
            if (coop && run) {
                atomicAdd(&expert_count[e], run);
                atomicAdd(&rank_sum[e / El], run);
            }
        }
        __syncthreads();
        if (coop && tid < R && rank_sum[tid]) atomicAdd(&splits_acc[s * R + tid], rank_sum[tid]);
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

    unsigned* counter = &hdr->done;
    int* bstart = reinterpret_cast<int*>(smem_raw);   // [kLWarps][R+1]
    int* ctot = bstart + kLWarps * (R + 1);            // [E]
    int* acc_splits = ctot + E;                        // [R*R]
    int* mat = acc_splits + R * R;                     // [E+R][n_tiles] when staged
    int* bs = bstart + warp * (R + 1);
    const int nrows = E + R;

    if (coop) {
        // ------- cooperative: one barrier, then phase 3 and phase 2 at once ---
        if (!grid_barrier(counter, gridDim.x + bar_extra, bar_limit_ns)) {
            if (tid == 0) atomicOr(status, MOE_ST_TIMEOUT);
            return;
        }
        const int G = gridDim.x;
        if (j == 0) {
            if (tid < E) {
                const int c = __ldcg(expert_count + tid);
                tokens_per_expert[tid] = c;
                ctot[tid] = ((c + align - 1) / align) * align;
            }
            for (int q = tid; q < R * R; q += kLThreads) splits[q] = __ldcg(splits_acc + q);
            __syncthreads();
            const int total = block_exclusive_scan_1024(ctot, E, scratch);
            if (tid < E) offsets[tid] = ctot[tid];
            if (tid == 0) offsets[E] = total;
            if (G > 1) return;
        }
        const int row_ctas = G > 1 ? G - 1 : 1;
        const int cta_rank = G > 1 ? j - 1 : 0;
        for (int p = cta_rank * kLWarps + warp; p < nrows; p += row_ctas * kLWarps)
            scan_row_regs(p, E, R, geo, tile_base, tile_tpr, bs, counts, tokens_per_rank);
        return;
    } else {
        // ------------------- the last CTA to arrive runs phases 2 and 3 ---
        __threadfence();
        __syncthreads();
        if (tid == 0) am_last = (atomicAdd(counter, 1u) == gridDim.x - 1);
        __syncthreads();
        if (!am_last) return;
        __threadfence();
        for (int q = tid; q < R * R; q += kLThreads) acc_splits[q] = 0;
        if (staged) {
            // Stage the whole count matrix (independent coalesced loads).
            const int ne = E * n_tiles, nr = R * n_tiles;
            for (int q = tid; q < ne; q += kLThreads) mat[q] = __ldcg(tile_base + q);
            for (int q = tid; q < nr; q += kLThreads) mat[ne + q] = __ldcg(tile_tpr + q);
        }
        __syncthreads();
        phases_2_3_one_cta(E, R, align, geo, staged ? mat : nullptr, bstart, ctot, acc_splits,
                           scratch, tile_base, tile_tpr, expert_count, tokens_per_expert, counts,
                           splits, tokens_per_rank, offsets);
    }
}

cudaError_t launch_layout(const int64_t* topk_idx, int T, int K, int E, int R, int align,
                          int32_t* tokens_per_expert, int32_t* counts, int32_t* splits,
                          int32_t* tokens_per_rank, uint8_t* is_token_in_rank,
                          int32_t* expert_offsets, void* workspace, int32_t* status,
                          cudaStream_t stream) {
    return launch_layout_ex(topk_idx, T, K, E, R, align, tokens_per_expert, counts, splits,
                            tokens_per_rank, is_token_in_rank, expert_offsets, workspace, status,
                            stream, 0u, kBarrierLimitNs, 0);
}

cudaError_t launch_layout_ex(const int64_t* topk_idx, int T, int K, int E, int R, int align,
                             int32_t* tokens_per_expert, int32_t* counts, int32_t* splits,
                             int32_t* tokens_per_rank, uint8_t* is_token_in_rank,
                             int32_t* expert_offsets, void* workspace, int32_t* status,
                             cudaStream_t stream, unsigned bar_extra, uint64_t bar_limit_ns,
                             int require_coop) {
    const Geometry geo = layout_geometry(T, K, R);
    const WsLayout wl = workspace_layout(E, R, geo.n_tiles, (int64_t)T * K);
    char* ws = static_cast<char*>(workspace);

    const int na_max = geo.TT * K;
    const size_t p1 = sizeof(unsigned long long) * geo.TT + sizeof(int) * na_max +
                      sizeof(uint16_t) * ((na_max + 1) & ~1) +
                      sizeof(uint16_t) * (size_t)((na_max + 31) / 32) * E;
    const size_t p2 = sizeof(int) * ((size_t)kLWarps * (R + 1) + E + (size_t)R * R);
    const size_t stage = sizeof(int) * (size_t)(E + R) * geo.n_tiles;
    const int staged = (p2 + stage) <= kLayoutSmemMax ? 1 : 0;
    const size_t p2s = p2 + (staged ? stage : 0);
    const size_t smem = p1 > p2s ? p1 : p2s;
    // Per-device caches (host threads may call concurrently: atomics).
    static std::atomic<int> configured[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    if (smem > 48 * 1024 &&
        (dev < 0 || dev >= 64 || configured[dev].load(std::memory_order_relaxed) < (int)smem)) {
        const cudaError_t e = cudaFuncSetAttribute(
            layout_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) {
            int cur = configured[dev].load(std::memory_order_relaxed);
            while (cur < (int)smem &&
                   !configured[dev].compare_exchange_weak(cur, (int)smem, std::memory_order_relaxed)) {
            }
        }
    }
    // Zero the arrival counter and the accumulators, then one launch:
    // cooperative (one grid barrier) when one CTA per tile fits on the GPU at
    // once, else last-CTA.
    cudaError_t err = cudaMemsetAsync(ws + wl.zero_begin, 0, wl.zero_end - wl.zero_begin, stream);
    if (err != cudaSuccess) return err;
    const int grid = geo.n_tiles > 0 ? geo.n_tiles : 1;
    int coop = (grid <= sm_count_current_device() && grid <= kCoopMaxTiles) ? 1 : 0;
    if (coop) {
        static std::atomic<int> coop_ok[64];
        if (dev >= 0 && dev < 64 && coop_ok[dev].load(std::memory_order_relaxed) == 0) {
            int attr = 0;
            if (cudaDeviceGetAttribute(&attr, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess)
                attr = 0;
            coop_ok[dev].store(attr ? 1 : -1, std::memory_order_relaxed);
        }
        if (dev < 0 || dev >= 64 || coop_ok[dev].load(std::memory_order_relaxed) != 1) coop = 0;
    }
    if (require_coop && !coop) return cudaErrorNotSupported;
    // With the barrier, phase 2 reads the rows from global memory: no staging.
    const int stg = coop ? 0 : staged;
    if (coop) {
        void* args[] = {(void*)&topk_idx, (void*)&T, (void*)&K, (void*)&E, (void*)&R,
                        (void*)&align, (void*)&geo, (void*)&tokens_per_expert, (void*)&counts,
                        (void*)&splits, (void*)&tokens_per_rank, (void*)&is_token_in_rank,
                        (void*)&expert_offsets, (void*)&ws, (void*)&wl, (void*)&status,
                        (void*)&coop, (void*)&stg, (void*)&bar_extra, (void*)&bar_limit_ns};
        return cudaLaunchCooperativeKernel((const void*)layout_kernel, dim3(grid), dim3(kLThreads),
                                           args, smem, stream);
    }
    layout_kernel<<<grid, kLThreads, smem, stream>>>(topk_idx, T, K, E, R, align, geo,
                                                     tokens_per_expert, counts, splits,
                                                     tokens_per_rank, is_token_in_rank,
                                                     expert_offsets, ws, wl, status, coop, stg,
                                                     bar_extra, bar_limit_ns);
    return cudaGetLastError();
}

}  // namespace moe
