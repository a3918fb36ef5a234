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
// pad rows.  Two kernels: for fan-out K >= 3 (and every payload permute),
// permute_kernel cuts the work into equal warp items (4 KB row pieces)
// strided over a grid of several CTAs per SM, so every warp moves the same
// bytes; for K <= 2, permute_ring_kernel streams each SM's share of the token
// rows through a deep ring of shared-memory buffers filled by bulk loads.
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

// ------------------------------------------------------ ring permute ---
//
// The same rows and maps again, for fan-out K <= 2, arranged so that
// a small problem has nearly all of its token rows in flight at once: one
// CTA per SM owns a contiguous range of token pieces (balanced to within one
// piece) and a ring of S 4 KB shared-memory buffers.  Thread 0 issues the
// first few bulk loads before anything else; the whole CTA then computes the
// rows of its tokens into shared memory (the owner of a token's first piece
// writes both maps) while they land; then thread 0 fills the rest of the ring
// and refills each buffer as soon as it is released.  Warps 1.. take the
// pieces in turn: wait for the piece, copy it to registers, release the
// buffer, store it to the token's K rows with 16-byte stores; afterwards they
// clear the pad rows and mark the tail.  Every mbarrier wait is bounded: on
// expiry the CTA records MOE_ST_TIMEOUT, waits (bounded) for its loads in
// flight and stops.
//
// Measured on B200 (Mixtral-shaped dispatch, 4096 tokens of 8 KB, eager
// permute): the whole ring requested first, 26.5 us (ncu: the layout reads
// the rows need queue behind 29 MB of loads; warps wait at the CTA barrier
// 44% of the time); 8, 4 or 2 pieces first, 21.7, 20.6 and 20.9 us; bulk
// stores issued by one thread instead of the consumer warps' stores, 45 us.
#ifndef MOE_RING_FIRST
#define MOE_RING_FIRST 4
#endif
constexpr int kRingFirst = MOE_RING_FIRST;   // pieces requested before the rows are known

template <int S>
struct RingSmem {
    static constexpr size_t rows = (size_t)S * kRingPiece;           // [kRingRows]
    static constexpr size_t ints = rows + sizeof(int) * kRingRows;   // off, padstart
    static size_t total(int E) { return ints + sizeof(int) * 2 * ((size_t)E + 1); }
};

template <int S>
__global__ void __launch_bounds__(kBlock, 1)
permute_ring_kernel(const char* __restrict__ x, int row_bytes, const int64_t* __restrict__ topk,
                    int T, int K, int E, const int32_t* __restrict__ offsets,
                    const char* __restrict__ ws, int zero_pad, int64_t N_cap, char* __restrict__ xp,
                    int32_t* __restrict__ r2f, int32_t* __restrict__ f2r,
                    int32_t* __restrict__ status) {
    static_assert(kRingFirst >= 1 && kRingFirst <= S, "the first batch fits the ring");
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ int scratch[kWarps + 1];
    __shared__ uint64_t full[S], empty[S];
    __shared__ int abort_flag, n_issued;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    unsigned char* ring = smem_raw;
    int* rows = reinterpret_cast<int*>(smem_raw + RingSmem<S>::rows);
    int* off = reinterpret_cast<int*>(smem_raw + RingSmem<S>::ints);   // [E+1]
    int* padstart = off + (E + 1);                                       // [E+1]

    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init_fence();
        abort_flag = 0;
        n_issued = 0;
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();
    const int pieces = (row_bytes + kRingPiece - 1) / kRingPiece;
    const int64_t tok_items = (int64_t)T * pieces;
    const int64_t i0 = tok_items * blockIdx.x / gridDim.x;
    const int64_t i1 = tok_items * (blockIdx.x + 1) / gridDim.x;
    const int n_my = (int)(i1 - i0);
    // Tokens this CTA's pieces belong to (the launch sizes the grid so that
    // they fit the row table).
    const int64_t t_lo = i0 / pieces;
    const int64_t t_hi = n_my > 0 ? (i1 + pieces - 1) / pieces : t_lo;
    if ((t_hi - t_lo) * K > kRingRows) {
        if (tid == 0) atomicOr(status, MOE_ST_LAYOUT_MISMATCH);
        return;
    }

    // Piece j of this CTA's range into buffer j % S.
    auto issue_load = [&](int j) {
        const int64_t item = i0 + j;
        const int64_t t = item / pieces;
        const int p = (int)(item - t * pieces);
        const unsigned bytes = (unsigned)min(kRingPiece, row_bytes - p * kRingPiece);
        mbar_expect_tx(&full[j % S], bytes);
        bulk_load(ring + (size_t)(j % S) * kRingPiece,
                  x + (size_t)t * row_bytes + (size_t)p * kRingPiece, bytes, &full[j % S]);
    };
    // The token rows do not depend on the layout: request the first few at
    // once, the rest of the ring once the rows are known (a full ring of
    // loads issued first delays the layout reads queued behind it).
    if (tid == 0) {
        const int first = min(kRingFirst, n_my);
        for (int j = 0; j < first; ++j) issue_load(j);
        n_issued = first;
    }
    const LayoutHeader* hdr = reinterpret_cast<const LayoutHeader*>(ws);
    if (hdr->magic != kLayoutMagic || hdr->T != T || hdr->K != K || hdr->E != E) {
        if (tid == 0) {
            if (blockIdx.x == 0) atomicOr(status, MOE_ST_LAYOUT_MISMATCH);
            for (int j = 0; j < n_issued; ++j)        // bounded wait for the loads in flight
                for (unsigned spins = 0; spins < kRingSpinLimit; ++spins)
                    if (mbar_try_wait(&full[j], 0u)) break;
        }
        return;
    }

    const int R = hdr->R, TT = hdr->TT, tpb = hdr->tpb, n_tiles = hdr->n_tiles;
    const int Tb = T / R;
    const int32_t* tile_base = reinterpret_cast<const int32_t*>(ws + hdr->off_tile_base);
    const int32_t* ecount = reinterpret_cast<const int32_t*>(ws + hdr->off_expert_count);
    const uint16_t* in_rank = reinterpret_cast<const uint16_t*>(ws + hdr->off_in_rank);
    // One round of independent loads: the offsets, the expert counts, and
    // the expert and in-tile rank of every row of this CTA's tokens (packed
    // e << 16 | rank into the row table, -1 for an expert out of range).
    constexpr int kOffPer = MOE_MAX_E / kBlock + 1;
    int offv[kOffPer], cntv[kOffPer];
#pragma unroll
    for (int c = 0; c < kOffPer; ++c) {
        const int e = tid + c * kBlock;
        offv[c] = e <= E ? offsets[e] : 0;
        cntv[c] = e < E ? ecount[e] : 0;
    }
    const int n_rows = (int)(t_hi - t_lo) * K;
    int bad = 0;
    for (int idx = tid; idx < n_rows; idx += kBlock) {
        const int64_t f = t_lo * K + idx;
        const int64_t e = topk[f];
        const int ir = in_rank[f];
        rows[idx] = (e >= 0 && e < E) ? (int)(e << 16) | ir : -1;
    }
#pragma unroll
    for (int c = 0; c < kOffPer; ++c) {
        const int e = tid + c * kBlock;
        if (e <= E) off[e] = offv[c];
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < kOffPer; ++c) {
        const int e = tid + c * kBlock;
        if (e < E) padstart[e] = (off[e + 1] - off[e]) - cntv[c];
    }
    __syncthreads();
    const int P = block_exclusive_scan<MOE_MAX_E / kBlock>(padstart, E, scratch);
    if (tid == 0) padstart[E] = P;
    const int64_t N_pad = off[E];
    if (blockIdx.x == 0 && tid == 0 && N_pad > N_cap) atomicOr(status, MOE_ST_CAPACITY);

    // Rows: off[e] + the tile's base + the in-tile rank; the owner of a
    // token's first piece writes both maps.
    for (int idx = tid; idx < n_rows; idx += kBlock) {
        const int64_t f = t_lo * K + idx;
        const int64_t t = f / K;
        const bool owner = t * pieces >= i0;
        const int packed = rows[idx];
        int myrow = -1;
        if (packed >= 0) {
            const int e = packed >> 16;
            const int s = (int)(t / Tb);
            const int jt = s * tpb + (int)(t - (int64_t)s * Tb) / TT;
            const int64_t row = (int64_t)off[e] + tile_base[(size_t)e * n_tiles + jt] + (packed & 0xFFFF);
            if (row >= 0 && row < N_cap) myrow = (int)row;
            else if (owner) bad |= MOE_ST_CAPACITY;
        } else if (owner) {
            bad |= MOE_ST_EXPERT_OOR;
        }
        rows[idx] = myrow;
        if (owner) {
            f2r[f] = myrow;
            if (myrow >= 0) r2f[myrow] = (int32_t)f;
        }
    }
    warp_status_or(status, bad);
    __syncthreads();

    if (warp == 0) {
        // Producer: fill the rest of the ring, then refill buffer j % S
        // once piece j - S has been copied out of it.
        if (lane == 0) {
            int j = n_issued;
            for (; j < min(S, n_my); ++j) issue_load(j);
            for (; j < n_my; ++j) {
                const unsigned parity = (unsigned)((j / S - 1) & 1);
                bool ok = false;
                for (unsigned spins = 0; spins < kRingSpinLimit; ++spins) {
                    if (mbar_try_wait(&empty[j % S], parity)) { ok = true; break; }
                    if (*(volatile int*)&abort_flag) break;
                }
                if (!ok) {
                    *(volatile int*)&abort_flag = 1;
                    break;
                }
                issue_load(j);
            }
            n_issued = j;
        }
    } else {
        // Consumers (warps 1..): piece j goes to warp 1 + j % (kWarps - 1);
        // shared memory -> registers (the buffer is released at once) ->
        // the token's K rows.
        const int cw = warp - 1, CW = kWarps - 1;
        const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
        for (int j = cw; j < n_my; j += CW) {
            bool ok = false;
            if (lane == 0) {
                const unsigned parity = (unsigned)((j / S) & 1);
                for (unsigned spins = 0; spins < kRingSpinLimit; ++spins) {
                    if (mbar_try_wait(&full[j % S], parity)) { ok = true; break; }
                    if (*(volatile int*)&abort_flag) break;
                }
                if (!ok) *(volatile int*)&abort_flag = 1;
            }
            if (!__shfl_sync(kFull, (int)ok, 0)) break;
            const int64_t item = i0 + j;
            const int64_t t = item / pieces;
            const int p = (int)(item - t * pieces);
            const int nv = min(kRingPiece, row_bytes - p * kRingPiece) / 16;
            const uint4* src = reinterpret_cast<const uint4*>(ring + (size_t)(j % S) * kRingPiece);
            uint4 v[kRingPiece / 16 / 32];
#pragma unroll
            for (int u = 0; u < kRingPiece / 16 / 32; ++u) v[u] = (lane + 32 * u < nv) ? src[lane + 32 * u] : zero;
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[j % S]);
            const int* trow = rows + (t - t_lo) * K;
            for (int k = 0; k < K; ++k) {
                const int r = trow[k];
                if (r < 0) continue;
                uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)r * row_bytes + (size_t)p * kRingPiece);
#pragma unroll
                for (int u = 0; u < kRingPiece / 16 / 32; ++u)
                    if (lane + 32 * u < nv) st_vec(dst + lane + 32 * u, v[u]);
            }
        }
        // Pad rows (one warp per row) and the tail of the row map.
        const int hw = blockIdx.x * CW + cw, HW = gridDim.x * CW;
        const int n16 = row_bytes / 16;
        for (int q = hw; q < P; q += HW) {
            const int e = upper_index(padstart, E + 1, q);
            const int64_t row = (int64_t)off[e] + ecount[e] + (q - padstart[e]);
            if (row < 0 || row >= N_cap) continue;
            if (lane == 0) r2f[row] = -1;
            if (!zero_pad) continue;
            uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)row * row_bytes);
            for (int v = lane; v < n16; v += 32) st_vec(dst + v, zero);
        }
        const int64_t tail0 = N_pad > 0 ? N_pad : 0;
        const int ht = hw * 32 + lane, HT = HW * 32;
        for (int64_t row = tail0 + ht; row < N_cap; row += HT) r2f[row] = -1;
    }
    __syncthreads();
    if (tid == 0 && abort_flag) {
        // Loads still in flight target this CTA's buffers (only the last S
        // issued can be): wait for them (bounded) before its shared memory
        // goes away.
        atomicOr(status, MOE_ST_TIMEOUT);
        for (int j = max(0, n_issued - S); j < n_issued; ++j)
            for (unsigned spins = 0; spins < kRingSpinLimit; ++spins)
                if (mbar_try_wait(&full[j % S], (unsigned)((j / S) & 1))) break;
    }
}

template <int S>
static cudaError_t launch_ring(const uint16_t* x, int row_bytes, const int64_t* topk_idx, int T,
                               int K, int E, const int32_t* expert_offsets, const void* workspace,
                               int zero_pad, int64_t N_cap, uint16_t* x_perm, int32_t* row_to_flat,
                               int32_t* flat_to_row, int32_t* status, cudaStream_t stream) {
    const size_t smem = RingSmem<S>::total(E);
    static std::atomic<int> configured[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    if (dev < 0 || dev >= 64 || configured[dev].load(std::memory_order_relaxed) < (int)smem) {
        const cudaError_t e = cudaFuncSetAttribute(
            permute_ring_kernel<S>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) {
            int cur = configured[dev].load(std::memory_order_relaxed);
            while (cur < (int)smem &&
                   !configured[dev].compare_exchange_weak(cur, (int)smem, std::memory_order_relaxed)) {
            }
        }
    }
    // One CTA per SM, more when a CTA's tokens would not fit its row table
    // (a range of n pieces spans at most n / pieces + 2 tokens; the caller
    // keeps K <= kRingRows / 4, so a CTA holds at least 2 whole tokens).
    const int sms = sm_count_current_device();
    const int64_t per_cta = kRingRows / K - 2;
    int64_t grid = ((int64_t)T + per_cta - 1) / per_cta;
    if (grid < sms) grid = sms;
    return launch_pdl(permute_ring_kernel<S>, dim3((int)grid), dim3(kBlock), smem, stream,
                      reinterpret_cast<const char*>(x), row_bytes, topk_idx, T, K, E,
                      expert_offsets, static_cast<const char*>(workspace), zero_pad, N_cap,
                      reinterpret_cast<char*>(x_perm), row_to_flat, flat_to_row, status);
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

cudaError_t launch_permute(const uint16_t* x, const int64_t* topk_idx, int T, int K, int E, int H,
                           const int32_t* expert_offsets, const void* workspace, int zero_pad,
                           int64_t N_cap, uint16_t* x_perm, int32_t* row_to_flat,
                           int32_t* flat_to_row, int32_t* status, cudaStream_t stream) {
    // Fan-out of at most 2 (each token row copied to <= 2 rows): the ring
    // kernel (measured on B200 against a copy-engine kernel with per-warp
    // two-stage buffers and bulk stores: Mixtral-shaped dispatch 49.5 vs
    // 51.4 us, the same at 32768 tokens 135.0 vs 138.4 us); larger fan-out:
    // the register kernel (the ring at fan-out 8: Qwen3-shaped permute 113.0
    // vs 97.4 us, DeepSeek-V3-shaped 237.5 vs 200.1 us).
#ifndef MOE_RING_S
#define MOE_RING_S 48
#endif
#ifndef MOE_RING_MAXK
#define MOE_RING_MAXK 2
#endif
    static_assert(MOE_RING_MAXK <= kRingRows / 4, "a CTA's row table holds two tokens");
    if (K <= MOE_RING_MAXK)
        return launch_ring<MOE_RING_S>(x, 2 * H, topk_idx, T, K, E, expert_offsets, workspace,
                                       zero_pad, N_cap, x_perm, row_to_flat, flat_to_row, status,
                                       stream);
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
