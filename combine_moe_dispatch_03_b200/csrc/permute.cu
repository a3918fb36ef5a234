// permute.cu -- dispatch on one device: token rows -> expert-grouped buffer.
//
// Source: the dispatch of the DeepEP issue "Does Deepep's Dispatch/Combine
// Support Autograd Like PyTorch's all_to_all?" and step 3 of the DeepSpeed
// AutoEP base PR (Design: "reorder tokens by expert assignment"), with the
// token-group padding of its Attribution section.
//
// Assignment f = (t, k) of expert e goes to row
//     off[e] + (assignments of e in earlier tiles) + (earlier in its tile)
// which is the stable (expert, token, slot) order.  All three terms are ready
// in the layout workspace (the per-tile bases after the scan and the
// in-tile ranks the histogram pass computed), so this is one streaming kernel:
// one read of every token row, K writes of it, the two row maps, and the
// pad rows.  Work is cut into equal warp items (4 KB row pieces) and strided
// over a grid of several CTAs per SM, so every warp moves the same bytes.
//
// Rows are opaque: a row is n16 16-byte vectors (bf16 rows: H/8; FP8 rows of
// the (data, scales) tuple the DeepEP issue's dispatch accepts: H/16; fp32
// rows: H/4).  With AUX, every token also owns a small aux row of 4-byte
// words (the FP8 scales) that goes to the same K rows.
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace moe {

// Grid-stride over warp items, all of one size: first (token, piece) items --
// a piece is 32 lanes x U 16-byte vectors of the token's row, read once and
// stored to the token's K rows -- then (pad row, piece) items.  The rows come
// from the layout workspace: row(f) = off[e] + tile_base[e][tile(t)] +
// in_rank[f]; the warp that handles piece 0 of a token also writes the
// token's entries of both maps (and, with AUX, copies the aux row).  A final
// sweep marks the tail rows.
// W32: every row is a whole number of 32-byte vectors in 32-byte-aligned
// buffers, and each lane moves U/2 32-byte vectors of the piece (two 16-byte
// vectors per instruction) instead of U 16-byte ones.
// MINB: resident CTAs per SM the registers are budgeted for.  With 4 the
// kernel spills a little (64 registers); with 3 it does not (about 80).
// Measured: 3 is faster at fan-out K >= 4 (Qwen3 and DeepSeek-V3 shapes),
// 4 at K = 2 (Mixtral shape).
template <int U, bool AUX, bool W32, int MINB>
__global__ void __launch_bounds__(kBlock, MINB)
permute_kernel(const uint4* __restrict__ x, int n16, const uint32_t* __restrict__ aux,
               int aux_words, const int64_t* __restrict__ topk, int T, int K, int E,
               const int32_t* __restrict__ offsets, const char* __restrict__ ws, int zero_pad,
               int64_t N_cap, uint4* __restrict__ xp, uint32_t* __restrict__ auxp,
               int32_t* __restrict__ r2f, int32_t* __restrict__ f2r,
               int32_t* __restrict__ status) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ int scratch[kWarps + 1];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();
    pdl_trigger();
    const LayoutHeader* hdr = reinterpret_cast<const LayoutHeader*>(ws);
    if (hdr->magic != kLayoutMagic || hdr->T != T || hdr->K != K || hdr->E != E) {
        if (blockIdx.x == 0 && tid == 0) atomicOr(status, MOE_ST_LAYOUT_MISMATCH);
        return;
    }
    const int R = hdr->R, TT = hdr->TT, tpb = hdr->tpb, n_tiles = hdr->n_tiles;
    const int Tb = T / R;
    const int32_t* tile_base = reinterpret_cast<const int32_t*>(ws + hdr->off_tile_base);
    const int32_t* ecount = reinterpret_cast<const int32_t*>(ws + hdr->off_expert_count);
    const uint16_t* in_rank = reinterpret_cast<const uint16_t*>(ws + hdr->off_in_rank);

    int* off = reinterpret_cast<int*>(smem_raw);   // [E+1]
    int* padstart = off + (E + 1);                  // [E+1]
    for (int e = tid; e <= E; e += kBlock) off[e] = offsets[e];
    __syncthreads();
    for (int e = tid; e < E; e += kBlock) padstart[e] = (off[e + 1] - off[e]) - ecount[e];
    __syncthreads();
    const int P = block_exclusive_scan<MOE_MAX_E / kBlock>(padstart, E, scratch);
    if (tid == 0) padstart[E] = P;
    __syncthreads();
    const int64_t N_pad = off[E];
    if (blockIdx.x == 0 && tid == 0 && N_pad > N_cap) atomicOr(status, MOE_ST_CAPACITY);

    const int pieces = (n16 + 32 * U - 1) / (32 * U);
    const int64_t tok_items = (int64_t)T * pieces;
    const int64_t n_items = tok_items + (int64_t)P * pieces;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    int bad = 0;

    for (int64_t item = (int64_t)blockIdx.x * kWarps + warp; item < n_items;
         item += (int64_t)gridDim.x * kWarps) {
        if (item < tok_items) {
            const int64_t t = item / pieces;
            const int p = (int)(item - t * pieces);
            // Lane's vectors of the piece: 16-byte vectors v0 + 32u, or with
            // W32 the pairs (v0 + 64u', v0 + 64u' + 1), v0 even.
            const int v0 = p * 32 * U + (W32 ? 2 * lane : lane);
            const uint4* src = x + (size_t)t * n16;
            uint4 v[U];
            if constexpr (W32) {
#pragma unroll
                for (int u = 0; u < U / 2; ++u) {
                    Vec32 w2 = make_vec32_zero();
                    if (v0 + 64 * u < n16) w2 = ld_stream32(src + v0 + 64 * u);
                    v[2 * u] = w2.lo;
                    v[2 * u + 1] = w2.hi;
                }
            } else {
#pragma unroll
                for (int u = 0; u < U; ++u) v[u] = (v0 + 32 * u < n16) ? ld_stream(src + v0 + 32 * u) : zero;
            }
            int myrow = -1;
            if (lane < K) {
                const int64_t f = t * K + lane;
                const int64_t e = topk[f];
                if (e >= 0 && e < E) {
                    const int s = (int)(t / Tb);
                    const int jt = s * tpb + (int)(t - (int64_t)s * Tb) / TT;
                    const int64_t row = (int64_t)off[e] + tile_base[(size_t)e * n_tiles + jt] + in_rank[f];
                    if (row >= 0 && row < N_cap) myrow = (int)row;
                    else if (p == 0) bad |= MOE_ST_CAPACITY;
                } else if (p == 0) {
                    bad |= MOE_ST_EXPERT_OOR;
                }
                if (p == 0) {
                    f2r[f] = myrow;
                    if (myrow >= 0) r2f[myrow] = (int32_t)f;
                }
            }
            for (int k = 0; k < K; ++k) {
                const int r = __shfl_sync(kFull, myrow, k);
                if (r < 0) continue;
                uint4* dst = xp + (size_t)r * n16;
                if constexpr (W32) {
#pragma unroll
                    for (int u = 0; u < U / 2; ++u)
                        if (v0 + 64 * u < n16) st_vec32(dst + v0 + 64 * u, Vec32{v[2 * u], v[2 * u + 1]});
                } else {
#pragma unroll
                    for (int u = 0; u < U; ++u)
                        if (v0 + 32 * u < n16) st_vec(dst + v0 + 32 * u, v[u]);
                }
                if (AUX && p == 0) {
                    const uint32_t* asrc = aux + (size_t)t * aux_words;
                    uint32_t* adst = auxp + (size_t)r * aux_words;
                    for (int q = lane; q < aux_words; q += 32) adst[q] = __ldg(asrc + q);
                }
            }
        } else {
            const int64_t pi = item - tok_items;
            const int q = (int)(pi / pieces);
            const int p = (int)(pi - (int64_t)q * pieces);
            const int v0 = p * 32 * U + (W32 ? 2 * lane : lane);
            const int e = upper_index(padstart, E + 1, q);
            const int64_t row = (int64_t)off[e] + ecount[e] + (q - padstart[e]);
            if (row < 0 || row >= N_cap) continue;
            if (p == 0 && lane == 0) r2f[row] = -1;
            if (!zero_pad) continue;
            if (AUX && p == 0)
                for (int wd = lane; wd < aux_words; wd += 32) auxp[(size_t)row * aux_words + wd] = 0u;
            uint4* dst = xp + (size_t)row * n16;
            if constexpr (W32) {
#pragma unroll
                for (int u = 0; u < U / 2; ++u)
                    if (v0 + 64 * u < n16) st_vec32(dst + v0 + 64 * u, make_vec32_zero());
            } else {
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (v0 + 32 * u < n16) st_vec(dst + v0 + 32 * u, zero);
            }
        }
    }
    warp_status_or(status, bad);

    const int64_t tail0 = N_pad > 0 ? N_pad : 0;
    for (int64_t row = tail0 + (int64_t)blockIdx.x * kBlock + tid; row < N_cap;
         row += (int64_t)gridDim.x * kBlock)
        r2f[row] = -1;
}

// ------------------------------------------------ bulk-copy permute ---
//
// The same items, rows and maps as permute_kernel (4 KB pieces of token rows,
// then pad-row pieces), moved by the copy engine instead of registers: per
// warp an S-stage pipeline of shared-memory buffers; lane 0 pulls a token
// piece into a buffer with one bulk load (completion on the buffer's
// mbarrier) and pushes it to the token's K rows with K bulk stores (one bulk
// group per item); pad pieces are pushed from a zeroed buffer.  Loads run
// S-1 items ahead; a buffer is reloaded only once the stores of the item
// that last used it have read it.  Every mbarrier wait is bounded: on expiry
// the warp records MOE_ST_TIMEOUT, waits (bounded) for its loads in flight
// and its stores, and stops.
//
// Used for fan-out K <= 2 only: measured on B200 it is slower than the
// register kernel at fan-out 8 (Qwen3 shape 113 vs 99 us, DeepSeek-V3 shape
// 238 vs 204 us) and a little faster at fan-out 2 (Mixtral shape, two
// stages: 21.8 vs 23.5 us).
constexpr int kBulkPiece = 4096;
constexpr unsigned kBulkSpinLimit = 1u << 22;

template <int S>
struct BulkSmem {
    static constexpr size_t zero = 0;
    static constexpr size_t bufs = kBulkPiece;                      // [kWarps][S][piece]
    static constexpr size_t bars = bufs + (size_t)kWarps * S * kBulkPiece;
    static constexpr size_t ints = bars + sizeof(uint64_t) * kWarps * S;   // off, padstart
    static size_t total(int E) { return ints + sizeof(int) * 2 * ((size_t)E + 1); }
};

template <int S>
__global__ void __launch_bounds__(kBlock)
permute_bulk_kernel(const char* __restrict__ x, int row_bytes, const int64_t* __restrict__ topk,
                    int T, int K, int E, const int32_t* __restrict__ offsets,
                    const char* __restrict__ ws, int zero_pad, int64_t N_cap, char* __restrict__ xp,
                    int32_t* __restrict__ r2f, int32_t* __restrict__ f2r,
                    int32_t* __restrict__ status) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ int scratch[kWarps + 1];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    unsigned char* zbuf = smem_raw + BulkSmem<S>::zero;
    unsigned char* mybuf = smem_raw + BulkSmem<S>::bufs + (size_t)warp * S * kBulkPiece;
    uint64_t* mybar = reinterpret_cast<uint64_t*>(smem_raw + BulkSmem<S>::bars) + warp * S;
    int* off = reinterpret_cast<int*>(smem_raw + BulkSmem<S>::ints);   // [E+1]
    int* padstart = off + (E + 1);                                      // [E+1]

    for (int i = tid; i < kBulkPiece / 16; i += kBlock)
        reinterpret_cast<uint4*>(zbuf)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (lane == 0) {
        for (int i = 0; i < S; ++i) mbar_init(&mybar[i], 1);
        mbar_init_fence();
    }
    fence_proxy_async_smem();
    pdl_wait();
    pdl_trigger();
    const LayoutHeader* hdr = reinterpret_cast<const LayoutHeader*>(ws);
    if (hdr->magic != kLayoutMagic || hdr->T != T || hdr->K != K || hdr->E != E) {
        if (blockIdx.x == 0 && tid == 0) atomicOr(status, MOE_ST_LAYOUT_MISMATCH);
        return;
    }
    const int R = hdr->R, TT = hdr->TT, tpb = hdr->tpb, n_tiles = hdr->n_tiles;
    const int Tb = T / R;
    const int32_t* tile_base = reinterpret_cast<const int32_t*>(ws + hdr->off_tile_base);
    const int32_t* ecount = reinterpret_cast<const int32_t*>(ws + hdr->off_expert_count);
    const uint16_t* in_rank = reinterpret_cast<const uint16_t*>(ws + hdr->off_in_rank);
    for (int e = tid; e <= E; e += kBlock) off[e] = offsets[e];
    __syncthreads();
    for (int e = tid; e < E; e += kBlock) padstart[e] = (off[e + 1] - off[e]) - ecount[e];
    __syncthreads();
    const int P = block_exclusive_scan<MOE_MAX_E / kBlock>(padstart, E, scratch);
    if (tid == 0) padstart[E] = P;
    __syncthreads();
    const int64_t N_pad = off[E];
    if (blockIdx.x == 0 && tid == 0 && N_pad > N_cap) atomicOr(status, MOE_ST_CAPACITY);

    const int pieces = (row_bytes + kBulkPiece - 1) / kBulkPiece;
    const int64_t tok_items = (int64_t)T * pieces;
    const int64_t n_items = tok_items + (int64_t)P * pieces;
    const int64_t gw = (int64_t)blockIdx.x * kWarps + warp, GW = (int64_t)gridDim.x * kWarps;
    const int64_t my_items = gw < n_items ? (n_items - gw + GW - 1) / GW : 0;
    int bad = 0;

    // Lane 0 issues the load of the warp's j-th item (token items only).
    auto issue_load = [&](int64_t j) {
        const int64_t item = gw + j * GW;
        if (item >= tok_items) return;
        const int64_t t = item / pieces;
        const int p = (int)(item - t * pieces);
        const unsigned bytes = (unsigned)min(kBulkPiece, row_bytes - p * kBulkPiece);
        uint64_t* bar = &mybar[j % S];
        mbar_expect_tx(bar, bytes);
        bulk_load(mybuf + (size_t)(j % S) * kBulkPiece,
                  x + (size_t)t * row_bytes + (size_t)p * kBulkPiece, bytes, bar);
    };
    if (lane == 0)
        for (int64_t j = 0; j < S - 1 && j < my_items; ++j) issue_load(j);

    int64_t j = 0;
    bool timed_out = false;
    for (; j < my_items; ++j) {
        const int64_t item = gw + j * GW;
        if (item < tok_items) {
            const int64_t t = item / pieces;
            const int p = (int)(item - t * pieces);
            const unsigned bytes = (unsigned)min(kBulkPiece, row_bytes - p * kBulkPiece);
            int myrow = -1;
            if (lane < K) {
                const int64_t f = t * K + lane;
                const int64_t e = topk[f];
                if (e >= 0 && e < E) {
                    const int s = (int)(t / Tb);
                    const int jt = s * tpb + (int)(t - (int64_t)s * Tb) / TT;
                    const int64_t row = (int64_t)off[e] + tile_base[(size_t)e * n_tiles + jt] + in_rank[f];
                    if (row >= 0 && row < N_cap) myrow = (int)row;
                    else if (p == 0) bad |= MOE_ST_CAPACITY;
                } else if (p == 0) {
                    bad |= MOE_ST_EXPERT_OOR;
                }
                if (p == 0) {
                    f2r[f] = myrow;
                    if (myrow >= 0) r2f[myrow] = (int32_t)f;
                }
            }
            // Wait for the piece (every lane polls, bounded); the warp
            // proceeds only if every lane saw it land.
            const unsigned parity = (unsigned)((j / S) & 1);
            bool landed = false;
            for (unsigned spins = 0; spins < kBulkSpinLimit; ++spins)
                if (mbar_try_wait(&mybar[j % S], parity)) { landed = true; break; }
            if (!__all_sync(kFull, landed)) {
                timed_out = true;
                break;
            }
            const unsigned char* src = mybuf + (size_t)(j % S) * kBulkPiece;
            for (int k = 0; k < K; ++k) {
                const int r = __shfl_sync(kFull, myrow, k);
                if (lane == 0 && r >= 0)
                    bulk_store(xp + (size_t)r * row_bytes + (size_t)p * kBulkPiece, src, bytes);
            }
        } else {
            const int64_t pi = item - tok_items;
            const int q = (int)(pi / pieces);
            const int p = (int)(pi - (int64_t)q * pieces);
            const unsigned bytes = (unsigned)min(kBulkPiece, row_bytes - p * kBulkPiece);
            const int e = upper_index(padstart, E + 1, q);
            const int64_t row = (int64_t)off[e] + ecount[e] + (q - padstart[e]);
            if (lane == 0 && row >= 0 && row < N_cap) {
                if (p == 0) r2f[row] = -1;
                if (zero_pad) bulk_store(xp + (size_t)row * row_bytes + (size_t)p * kBulkPiece, zbuf, bytes);
            }
        }
        if (lane == 0) {
            bulk_commit();
            // The buffer of item j+S-1 was last read by item j-1's stores.
            bulk_wait_read<1>();
            if (j + S - 1 < my_items) issue_load(j + S - 1);
        }
        __syncwarp();
    }
    if (timed_out) {
        // Loads in flight target this warp's buffers: wait for them (bounded)
        // before the CTA's shared memory goes away.
        bad |= MOE_ST_TIMEOUT;
        for (int64_t jj = j; jj < my_items && jj < j + S - 1; ++jj) {
            if (gw + jj * GW >= tok_items) continue;
            for (unsigned spins = 0; spins < kBulkSpinLimit; ++spins)
                if (mbar_try_wait(&mybar[jj % S], (unsigned)((jj / S) & 1))) break;
        }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
    warp_status_or(status, bad);

    const int64_t tail0 = N_pad > 0 ? N_pad : 0;
    for (int64_t row = tail0 + (int64_t)blockIdx.x * kBlock + tid; row < N_cap;
         row += (int64_t)gridDim.x * kBlock)
        r2f[row] = -1;
}

template <bool AUX>
static cudaError_t launch_rows(const uint4* x, int n16, const uint32_t* aux, int aux_words,
                               const int64_t* topk_idx, int T, int K, int E,
                               const int32_t* expert_offsets, const void* workspace, int zero_pad,
                               int64_t N_cap, uint4* x_perm, uint32_t* aux_perm,
                               int32_t* row_to_flat, int32_t* flat_to_row, int32_t* status,
                               cudaStream_t stream) {
    // Enough CTAs to fill every SM several times over; the kernel strides
    // over its uniform items (token pieces, then pad-row pieces <= N_cap - A).
#ifndef MOE_PERMUTE_U
#define MOE_PERMUTE_U 8
#endif
    constexpr int U = MOE_PERMUTE_U;
    const int sms = sm_count_current_device();
    const int64_t pieces = (n16 + 32 * U - 1) / (32 * U);
    const int64_t items = ((int64_t)T + (N_cap - (int64_t)T * K)) * pieces;
    int64_t grid = (items + kWarps - 1) / kWarps;
#ifndef MOE_PERMUTE_GRID_PER_SM
#define MOE_PERMUTE_GRID_PER_SM 32
#endif
    if (grid > (int64_t)sms * MOE_PERMUTE_GRID_PER_SM) grid = (int64_t)sms * MOE_PERMUTE_GRID_PER_SM;
    if (grid < 1) grid = 1;
#ifndef MOE_PERMUTE_W32
#define MOE_PERMUTE_W32 1
#endif
    const bool w32 = MOE_PERMUTE_W32 && (n16 % 2) == 0 &&
                     (reinterpret_cast<uintptr_t>(x) % 32) == 0 &&
                     (reinterpret_cast<uintptr_t>(x_perm) % 32) == 0;
    const size_t smem = sizeof(int) * 2 * ((size_t)E + 1);
#define MOE_PERMUTE_LAUNCH(W, M)                                                                 \
    launch_pdl(permute_kernel<U, AUX, W, M>, dim3((int)grid), dim3(kBlock), smem, stream, x, n16, \
               aux, aux_words, topk_idx, T, K, E, expert_offsets,                                 \
               static_cast<const char*>(workspace), zero_pad, N_cap, x_perm, aux_perm,           \
               row_to_flat, flat_to_row, status)
    if (K >= 4) return w32 ? MOE_PERMUTE_LAUNCH(true, 3) : MOE_PERMUTE_LAUNCH(false, 3);
    return w32 ? MOE_PERMUTE_LAUNCH(true, 4) : MOE_PERMUTE_LAUNCH(false, 4);
#undef MOE_PERMUTE_LAUNCH
}

template <int S>
static cudaError_t launch_bulk(const uint16_t* x, int row_bytes, const int64_t* topk_idx, int T,
                               int K, int E, const int32_t* expert_offsets, const void* workspace,
                               int zero_pad, int64_t N_cap, uint16_t* x_perm, int32_t* row_to_flat,
                               int32_t* flat_to_row, int32_t* status, cudaStream_t stream) {
    const size_t smem = BulkSmem<S>::total(E);
    // Per-device caches: the shared-memory opt-in set so far, and the
    // resident CTAs per SM at that size (host threads may call concurrently).
    static std::atomic<int> configured[64];
    static std::atomic<int> resident[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    int per_sm = 0;
    if (dev < 0 || dev >= 64 || configured[dev].load(std::memory_order_relaxed) < (int)smem) {
        const cudaError_t e = cudaFuncSetAttribute(
            permute_bulk_kernel<S>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, permute_bulk_kernel<S>, kBlock,
                                                          smem) != cudaSuccess)
            per_sm = 0;
        if (dev >= 0 && dev < 64) {
            int cur = configured[dev].load(std::memory_order_relaxed);
            while (cur < (int)smem &&
                   !configured[dev].compare_exchange_weak(cur, (int)smem, std::memory_order_relaxed)) {
            }
            resident[dev].store(per_sm, std::memory_order_relaxed);
        }
    } else {
        per_sm = resident[dev].load(std::memory_order_relaxed);
    }
    if (per_sm < 1) per_sm = 1;
    const int sms = sm_count_current_device();
    const int64_t pieces = (row_bytes + kBulkPiece - 1) / kBulkPiece;
    const int64_t items = ((int64_t)T + (N_cap - (int64_t)T * K)) * pieces;
    int64_t grid = (items + kWarps - 1) / kWarps;
    if (grid > (int64_t)sms * per_sm) grid = (int64_t)sms * per_sm;
    if (grid < 1) grid = 1;
    return launch_pdl(permute_bulk_kernel<S>, dim3((int)grid), dim3(kBlock), smem, stream,
                      reinterpret_cast<const char*>(x), row_bytes, topk_idx, T, K, E,
                      expert_offsets, static_cast<const char*>(workspace), zero_pad, N_cap,
                      reinterpret_cast<char*>(x_perm), row_to_flat, flat_to_row, status);
}

cudaError_t launch_permute(const uint16_t* x, const int64_t* topk_idx, int T, int K, int E, int H,
                           const int32_t* expert_offsets, const void* workspace, int zero_pad,
                           int64_t N_cap, uint16_t* x_perm, int32_t* row_to_flat,
                           int32_t* flat_to_row, int32_t* status, cudaStream_t stream) {
    // Fan-out of at most 2 (each token row copied to <= 2 rows): the bulk-copy
    // kernel measured faster (Mixtral shape 21.8 vs 23.5 us); larger fan-out:
    // the register kernel.
    if (K <= 2)
        return launch_bulk<2>(x, 2 * H, topk_idx, T, K, E, expert_offsets, workspace, zero_pad,
                              N_cap, x_perm, row_to_flat, flat_to_row, status, stream);
    return launch_rows<false>(reinterpret_cast<const uint4*>(x), H >> 3, nullptr, 0, topk_idx, T,
                              K, E, expert_offsets, workspace, zero_pad, N_cap,
                              reinterpret_cast<uint4*>(x_perm), nullptr, row_to_flat, flat_to_row,
                              status, stream);
}

cudaError_t launch_permute_payload(const void* x, int64_t row_bytes, const void* aux,
                                   int64_t aux_row_bytes, const int64_t* topk_idx, int T, int K,
                                   int E, const int32_t* expert_offsets, const void* workspace,
                                   int zero_pad, int64_t N_cap, void* x_perm, void* aux_perm,
                                   int32_t* row_to_flat, int32_t* flat_to_row, int32_t* status,
                                   cudaStream_t stream) {
    const int n16 = (int)(row_bytes / 16);
    const uint4* xs = static_cast<const uint4*>(x);
    uint4* xd = static_cast<uint4*>(x_perm);
    if (aux_row_bytes > 0 && aux_perm != nullptr)
        return launch_rows<true>(xs, n16, static_cast<const uint32_t*>(aux),
                                 (int)(aux_row_bytes / 4), topk_idx, T, K, E, expert_offsets,
                                 workspace, zero_pad, N_cap, xd, static_cast<uint32_t*>(aux_perm),
                                 row_to_flat, flat_to_row, status, stream);
    return launch_rows<false>(xs, n16, nullptr, 0, topk_idx, T, K, E, expert_offsets, workspace,
                              zero_pad, N_cap, xd, nullptr, row_to_flat, flat_to_row, status,
                              stream);
}

}  // namespace moe
