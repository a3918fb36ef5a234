// ranks.cu -- dispatch and combine straight into / out of the destination
// ranks' buffers, the fused form of expert parallelism across GPUs: instead
// of permuting into a local send buffer and handing it to an all-to-all, the
// permute stores every row into the receive buffer of the rank that owns its
// expert, and the combine gathers every slot's expert output from the buffer
// of the rank that computed it.  The buffers are reached through a device
// array of pointers, one per rank; across GPUs these are peer addresses
// (NVLink; plain loads and stores, no multicast), on one GPU they may be
// ordinary buffers.  Source: DeepEP issue "Does Deepep's Dispatch/Combine
// Support Autograd Like PyTorch's all_to_all?" (dispatch sends token rows to
// the ranks that own their experts; combine reduces them back) and DeepSpeed
// PR "Derive AutoEP rank splits from the per-expert count exchange" (the
// per-(source rank, expert) counts every rank derives its offsets from).
//
// The destination row of assignment f = (t, k) of expert e, sent by rank s,
// is dest_base[e] + (earlier assignments of e among s's own tokens, from the
// layout workspace of s's tokens), where dest_base[e] = (start of e's group
// in its owner's buffer) + (rows of e from ranks before s): the receive
// buffer of every rank comes out in the order the single-device layout gives
// those experts (source rank, token, slot), with the same padding.
#include "common.cuh"
#include "internal.h"

namespace moe {

// Token items as in permute_kernel, each slot's row going to the buffer of
// its expert's rank; then the pad rows of this rank's own receive buffer
// (own_offsets / own_counts of its E_local experts), zeroed.
template <int U>
__global__ void __launch_bounds__(kBlock, 4)
permute_to_ranks_kernel(const uint4* __restrict__ x, int n16, const int64_t* __restrict__ topk,
                        int T, int K, int E, int El, int R, const int32_t* __restrict__ dest_base,
                        const char* __restrict__ ws, uint4* const* __restrict__ dest,
                        int32_t* const* __restrict__ claims, int64_t dest_cap, int my_rank,
                        const int32_t* __restrict__ own_off, const int32_t* __restrict__ own_cnt,
                        int zero_pad, int32_t* __restrict__ f2r, int32_t* __restrict__ status) {
    __shared__ int padstart[MOE_MAX_E + 1];
    __shared__ int scratch[kWarps + 1];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();
    pdl_trigger();
    const LayoutHeader* hdr = reinterpret_cast<const LayoutHeader*>(ws);
    if (hdr->magic != kLayoutMagic || hdr->T != T || hdr->K != K || hdr->E != E || hdr->R != 1) {
        if (blockIdx.x == 0 && tid == 0) atomicOr(status, MOE_ST_LAYOUT_MISMATCH);
        return;
    }
    const int TT = hdr->TT, n_tiles = hdr->n_tiles;
    const int32_t* tile_base = reinterpret_cast<const int32_t*>(ws + hdr->off_tile_base);
    const uint16_t* in_rank = reinterpret_cast<const uint16_t*>(ws + hdr->off_in_rank);

    // Pad rows of this rank's own buffer: expert el has
    // own_off[el+1] - own_off[el] - own_cnt[el] of them after its real rows.
    for (int el = tid; el < El; el += kBlock) {
        const int p = (own_off[el + 1] - own_off[el]) - own_cnt[el];
        padstart[el] = p > 0 ? p : 0;
    }
    __syncthreads();
    const int P = block_exclusive_scan<MOE_MAX_E / kBlock>(padstart, El, scratch);
    if (tid == 0) padstart[El] = P;
    __syncthreads();

    const int pieces = (n16 + 32 * U - 1) / (32 * U);
    const int64_t tok_items = (int64_t)T * pieces;
    const int64_t n_items = tok_items + (zero_pad ? (int64_t)P * pieces : 0);
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
            int myrow = -1, myrank = 0;
            if (lane < K) {
                const int64_t f = t * K + lane;
                const int64_t e = topk[f];
                if (e >= 0 && e < E) {
                    const int jt = (int)(t / TT);
                    const int64_t row = (int64_t)dest_base[e] + tile_base[(size_t)e * n_tiles + jt] +
                                        in_rank[f];
                    if (row >= 0 && row < dest_cap) {
                        myrow = (int)row;
                        myrank = (int)(e / El);
                    } else if (p == 0) {
                        bad |= MOE_ST_CAPACITY;
                    }
                } else if (p == 0) {
                    bad |= MOE_ST_EXPERT_OOR;
                }
                if (p == 0) {
                    f2r[f] = myrow;
                    if (claims && myrow >= 0) claims[myrank][myrow] = claim_code(my_rank, f);
                }
            }
            for (int k = 0; k < K; ++k) {
                const int r = __shfl_sync(kFull, myrow, k);
                const int rk = __shfl_sync(kFull, myrank, k);
                if (r < 0) continue;
                uint4* dst = dest[rk] + (size_t)r * n16;
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (v0 + 32 * u < n16) st_vec(dst + v0 + 32 * u, v[u]);
            }
        } else {
            const int64_t pi = item - tok_items;
            const int q = (int)(pi / pieces);
            const int p = (int)(pi - (int64_t)q * pieces);
            const int v0 = p * 32 * U + lane;
            const int el = upper_index(padstart, El + 1, q);
            const int64_t row = (int64_t)own_off[el] + own_cnt[el] + (q - padstart[el]);
            if (row < 0 || row >= dest_cap) continue;
            uint4* dst = dest[my_rank] + (size_t)row * n16;
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (v0 + 32 * u < n16) st_vec(dst + v0 + 32 * u, zero);
        }
    }
    // Claims of this rank's own buffer that no sender writes this call (its
    // pad rows and the rows past its padded total) are cleared, so a stale
    // row never passes the restore's check.
    if (claims) {
        int32_t* mine = claims[my_rank];
        const int64_t gstride = (int64_t)gridDim.x * kBlock;
        const int64_t g0 = (int64_t)blockIdx.x * kBlock + tid;
        for (int64_t q = g0; q < P; q += gstride) {
            const int el = upper_index(padstart, El + 1, (int)q);
            const int64_t row = (int64_t)own_off[el] + own_cnt[el] + (q - padstart[el]);
            if (row >= 0 && row < dest_cap) mine[row] = -1;
        }
        for (int64_t row = (int64_t)own_off[El] + g0; row < dest_cap; row += gstride) mine[row] = -1;
    }
    warp_status_or(status, bad);
}

// One warp per token: for every column chunk the slots are visited in order
// and each slot's row is read from the buffer of its expert's rank; the same
// FP32 chain as combine_kernel, so the output is bit-identical to the
// single-device restore of the same rows.
template <int U>
__global__ void __launch_bounds__(kBlock)
combine_from_ranks_kernel(const uint4* const* __restrict__ rows,
                          const int32_t* const* __restrict__ claims, int my_rank, int R,
                          int64_t N_cap, const int32_t* __restrict__ f2r,
                          const int64_t* __restrict__ topk, int E, int El,
                          const void* __restrict__ w, int wdtype, int T, int K, int n16,
                          uint4* __restrict__ out, int32_t* __restrict__ status) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    pdl_wait();
    pdl_trigger();
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    int bad = 0;
    for (int t = blockIdx.x * kWarps + warp; t < T; t += gridDim.x * kWarps) {
        int myrow = -1, myrank = 0;
        float myw = 0.f;
        if (lane < K) {
            const int64_t f = (int64_t)t * K + lane;
            const int r = f2r[f];
            const int64_t e = topk[f];
            if (r < 0 || (int64_t)r >= N_cap || e < 0 || e >= E) {
                bad |= MOE_ST_ROW_OOR;
            } else {
                myrow = r;
                myrank = (int)(e / El);
                myw = load_weight(w, wdtype, f);
                if (claims && claims[myrank][r] != claim_code(my_rank, f)) bad |= MOE_ST_COVERAGE;
            }
        }
        uint4* dst = out + (size_t)t * n16;
        for (int c0 = 0; c0 < n16; c0 += 32 * U) {      // warp-uniform trip count
            const int c = c0 + lane;
            float acc[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;
            for (int k = 0; k < K; ++k) {
                const int r = __shfl_sync(kFull, myrow, k);
                const int rk = __shfl_sync(kFull, myrank, k);
                const float wv = __shfl_sync(kFull, myw, k);
                if (r < 0) continue;
                const uint4* src = rows[rk] + (size_t)r * n16;
                uint4 v[U];
#pragma unroll
                for (int u = 0; u < U; ++u) v[u] = (c + 32 * u < n16) ? ld_stream(src + c + 32 * u) : zero;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    float y[8];
                    unpack8(v[u], y);
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[u][i] = __fmaf_rn(wv, y[i], acc[u][i]);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (c + 32 * u < n16) st_vec(dst + c + 32 * u, pack8(acc[u]));
        }
    }
    warp_status_or(status, bad);
}

// Row bases of the direct dispatch from the per-expert counts of every
// source rank (all_counts [R][E]): one CTA.  Each thread takes experts e,
// sums the column over the source ranks (total) and over the ranks before
// `rank` (before); one CTA scan of the padded totals over all experts gives
// every group's start, and an owner's groups start at the scan value of its
// first expert, so
//   dest_base[e]    = scan[e] - scan[owner(e)*El] + before[e]
//   own_offsets[el] = scan[rank*El + el] - scan[rank*El]
//   max_rows        = max over owners r of scan[(r+1)*El] - scan[r*El].
__global__ void __launch_bounds__(kBlock)
rank_bases_kernel(const int32_t* __restrict__ all_counts, int R, int E, int rank, int align,
                  int32_t* __restrict__ dest_base, int32_t* __restrict__ own_off,
                  int32_t* __restrict__ own_cnt, int32_t* __restrict__ max_rows,
                  int32_t* __restrict__ status) {
    __shared__ int scan[MOE_MAX_E + 1];
    __shared__ int total[MOE_MAX_E];
    __shared__ int before[MOE_MAX_E];
    __shared__ int scratch[kWarps + 1];
    __shared__ int best;
    const int tid = threadIdx.x;
    const int El = E / R;
    pdl_wait();
    pdl_trigger();
    int bad = 0;
    if (tid == 0) best = 0;
    for (int e = tid; e < E; e += kBlock) {
        int64_t tot = 0, bef = 0;
        for (int s = 0; s < R; ++s) {
            int64_t c = all_counts[(size_t)s * E + e];
            if (c < 0) {
                bad |= MOE_ST_COVERAGE;
                c = 0;
            }
            tot += c;
            if (s < rank) bef += c;
        }
        const int64_t padded = (tot + align - 1) / align * align;
        if (padded > (int64_t)(INT32_MAX / MOE_MAX_E)) bad |= MOE_ST_CAPACITY;
        total[e] = (int)tot;
        before[e] = (int)bef;
        scan[e] = (int)padded;
    }
    __syncthreads();
    const int grand = block_exclusive_scan<MOE_MAX_E / kBlock>(scan, E, scratch);
    if (tid == 0) scan[E] = grand;
    __syncthreads();
    for (int e = tid; e < E; e += kBlock)
        dest_base[e] = scan[e] - scan[(e / El) * El] + before[e];
    const int mine = rank * El;
    for (int el = tid; el <= El; el += kBlock) {
        own_off[el] = scan[mine + el] - scan[mine];
        if (el < El) own_cnt[el] = total[mine + el];
    }
    for (int r = tid; r < R; r += kBlock) atomicMax(&best, scan[(r + 1) * El] - scan[r * El]);
    __syncthreads();
    if (tid == 0) *max_rows = best;
    warp_status_or(status, bad);
}

cudaError_t launch_rank_bases(const int32_t* all_counts, int R, int E, int rank, int align,
                              int32_t* dest_base, int32_t* own_offsets, int32_t* own_counts,
                              int32_t* max_rows, int32_t* status, cudaStream_t stream) {
    return launch_pdl(rank_bases_kernel, dim3(1), dim3(kBlock), 0, stream, all_counts, R, E, rank,
                      align, dest_base, own_offsets, own_counts, max_rows, status);
}

cudaError_t launch_permute_to_ranks(const uint16_t* x, const int64_t* topk_idx, int T, int K,
                                    int E, int R, int H, const int32_t* dest_base,
                                    const void* workspace, uint16_t* const* dest_rows,
                                    int32_t* const* dest_claims, int64_t dest_cap, int rank,
                                    const int32_t* own_offsets, const int32_t* own_counts,
                                    int zero_pad, int32_t* flat_to_row, int32_t* status,
                                    cudaStream_t stream) {
    constexpr int U = 8;
    const int n16 = H / 8;
    const int El = E / R;
    const int sms = sm_count_current_device();
    const int64_t pieces = (n16 + 32 * U - 1) / (32 * U);
    // token items plus at most El * (rows of the largest possible pad) pad items
    int64_t grid = ((int64_t)T * pieces + kWarps - 1) / kWarps + 1;
    if (grid > (int64_t)sms * 32) grid = (int64_t)sms * 32;
    if (grid < (int64_t)sms) grid = sms;
    return launch_pdl(permute_to_ranks_kernel<U>, dim3((int)grid), dim3(kBlock), 0, stream,
                      reinterpret_cast<const uint4*>(x), n16, topk_idx, T, K, E, El, R, dest_base,
                      static_cast<const char*>(workspace),
                      reinterpret_cast<uint4* const*>(dest_rows), dest_claims, dest_cap, rank,
                      own_offsets, own_counts, zero_pad, flat_to_row, status);
}

cudaError_t launch_combine_from_ranks(const uint16_t* const* rows, const int32_t* const* claims,
                                      int R, int rank, int64_t N_cap, const int32_t* flat_to_row,
                                      const int64_t* topk_idx, int E, const void* weights,
                                      int weight_dtype, int T, int K, int H, uint16_t* out,
                                      int32_t* status, cudaStream_t stream) {
    // K <= 8: the slot-major restore of combine.cu (contiguous row chunks,
    // several in flight per warp) reading each slot from its rank's buffer.
    if (K <= 8)
        return launch_combine_slots_from_ranks(rows, claims, R, rank, N_cap, flat_to_row, topk_idx,
                                               E, weights, weight_dtype, T, K, H, out, status,
                                               stream);
    constexpr int U = 2;
    const int sms = sm_count_current_device();
    int64_t grid = ((int64_t)T + kWarps - 1) / kWarps;
    if (grid > (int64_t)sms * 8) grid = (int64_t)sms * 8;
    if (grid < 1) grid = 1;
    return launch_pdl(combine_from_ranks_kernel<U>, dim3((int)grid), dim3(kBlock), 0, stream,
                      reinterpret_cast<const uint4* const*>(rows), claims, rank, R, N_cap,
                      flat_to_row, topk_idx, E, E / R, weights, weight_dtype, T, K, H / 8,
                      reinterpret_cast<uint4*>(out), status);
}

}  // namespace moe
