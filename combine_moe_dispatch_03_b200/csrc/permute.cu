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
template <int U, bool AUX>
__global__ void __launch_bounds__(kBlock, 4)
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
            const int v0 = p * 32 * U + lane;
            const uint4* src = x + (size_t)t * n16;
            uint4 v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) v[u] = (v0 + 32 * u < n16) ? ld_stream(src + v0 + 32 * u) : zero;
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
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (v0 + 32 * u < n16) st_vec(dst + v0 + 32 * u, v[u]);
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
            const int v0 = p * 32 * U + lane;
            const int e = upper_index(padstart, E + 1, q);
            const int64_t row = (int64_t)off[e] + ecount[e] + (q - padstart[e]);
            if (row < 0 || row >= N_cap) continue;
            if (p == 0 && lane == 0) r2f[row] = -1;
            if (!zero_pad) continue;
            if (AUX && p == 0)
                for (int wd = lane; wd < aux_words; wd += 32) auxp[(size_t)row * aux_words + wd] = 0u;
            uint4* dst = xp + (size_t)row * n16;
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (v0 + 32 * u < n16) st_vec(dst + v0 + 32 * u, zero);
        }
    }
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
    return launch_pdl(permute_kernel<U, AUX>, dim3((int)grid), dim3(kBlock),
                      sizeof(int) * 2 * ((size_t)E + 1), stream, x, n16, aux, aux_words, topk_idx,
                      T, K, E, expert_offsets, static_cast<const char*>(workspace), zero_pad,
                      N_cap, x_perm, aux_perm, row_to_flat, flat_to_row, status);
}

cudaError_t launch_permute(const uint16_t* x, const int64_t* topk_idx, int T, int K, int E, int H,
                           const int32_t* expert_offsets, const void* workspace, int zero_pad,
                           int64_t N_cap, uint16_t* x_perm, int32_t* row_to_flat,
                           int32_t* flat_to_row, int32_t* status, cudaStream_t stream) {
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
