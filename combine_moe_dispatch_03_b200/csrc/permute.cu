// permute.cu -- dispatch on one device: token rows -> expert-grouped buffer.
//
// Source: the dispatch of the DeepEP issue "Does Deepep's Dispatch/Combine
// Support Autograd Like PyTorch's all_to_all?" and step 3 of the DeepSpeed
// AutoEP base PR (Design: "reorder tokens by expert assignment"), with the
// token-group padding of its Attribution section.
//
// Assignment f = (t, k) of expert e goes to row
//     off[e] + (assignments of e in earlier tiles) + (earlier in this tile)
// which is the stable (expert, token, slot) order.  The first two terms come
// from the layout workspace; the in-tile rank is computed by one warp walking
// the tile's assignments in flat order, 32 at a time, with __match_any_sync
// giving each lane the lanes that share its expert.
//
// Data movement (the cost: one read of x, K writes of every row): one warp per
// token holds U 16-byte vectors per lane in registers and stores them to the
// K destination rows, so x is read from HBM exactly once and every store is a
// full, aligned, coalesced 512-byte warp transaction.  CTAs are persistent
// over tiles (grid <= SMs x resident CTAs), then share the pad rows evenly.
#include "common.cuh"
#include "internal.h"

namespace moe {

template <int U>
__global__ void __launch_bounds__(kBlock)
permute_kernel(const uint16_t* __restrict__ x, const int64_t* __restrict__ topk, int T, int K,
               int E, int H, const int32_t* __restrict__ offsets, const char* __restrict__ ws,
               int zero_pad, int64_t N_cap, uint16_t* __restrict__ xp,
               int32_t* __restrict__ r2f, int32_t* __restrict__ f2r,
               int32_t* __restrict__ status) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ int scratch[kWarps + 1];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    const LayoutHeader* hdr = reinterpret_cast<const LayoutHeader*>(ws);
    if (hdr->magic != kLayoutMagic || hdr->T != T || hdr->K != K || hdr->E != E) {
        if (blockIdx.x == 0 && tid == 0) atomicOr(status, MOE_ST_LAYOUT_MISMATCH);
        return;
    }
    const int R = hdr->R, TT = hdr->TT, tpb = hdr->tpb, n_tiles = hdr->n_tiles;
    const int32_t* tile_base = reinterpret_cast<const int32_t*>(ws + hdr->off_tile_base);
    const int32_t* ecount = reinterpret_cast<const int32_t*>(ws + hdr->off_expert_count);

    int* base = reinterpret_cast<int*>(smem_raw);   // [E+1]
    int* eidx = base + (E + 1);                      // [TT*K]
    int* rowi = eidx + TT * K;                       // [TT*K]

    const int64_t N_pad = offsets[E];
    if (blockIdx.x == 0 && tid == 0 && N_pad > N_cap) atomicOr(status, MOE_ST_CAPACITY);
    const int Tb = T / R;
    const int n16 = H >> 3;
    int bad = 0;

    for (int j = blockIdx.x; j < n_tiles; j += gridDim.x) {
        const int s = j / tpb, i = j - s * tpb;
        const int t0 = s * Tb + i * TT;
        const int t1 = min(t0 + TT, (s + 1) * Tb);
        const int ntok = t1 - t0, na = ntok * K;

        for (int e = tid; e < E; e += kBlock) base[e] = offsets[e] + tile_base[(size_t)e * n_tiles + j];
        for (int a = tid; a < na; a += kBlock) {
            const int64_t v = topk[(int64_t)t0 * K + a];
            eidx[a] = (v >= 0 && v < E) ? (int)v : -1;
        }
        __syncthreads();

        if (warp == 0) {
            const unsigned lt = lanemask_lt();
            for (int c0 = 0; c0 < na; c0 += 32) {
                const int a = c0 + lane;
                const int e = (a < na) ? eidx[a] : -1;
                const int key = (e >= 0) ? e : (-1 - lane);
                const unsigned peers = __match_any_sync(kFull, key);
                int row = -1;
                if (e >= 0) row = base[e] + __popc(peers & lt);
                __syncwarp();
                if (e >= 0 && lane == __ffs(peers) - 1) base[e] += __popc(peers);
                __syncwarp();
                if (a < na) {
                    const int64_t f = (int64_t)t0 * K + a;
                    const bool placed = (row >= 0) && ((int64_t)row < N_cap);
                    rowi[a] = placed ? row : -1;
                    f2r[f] = placed ? row : -1;
                    if (placed) r2f[row] = (int32_t)f;
                    if (e < 0) bad |= MOE_ST_EXPERT_OOR;
                    else if (!placed) bad |= MOE_ST_CAPACITY;
                }
            }
        }
        __syncthreads();

        // ---- copies: one warp per token, K stores per loaded vector ----
        for (int q = warp; q < ntok; q += kWarps) {
            const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(t0 + q) * H);
            const int myrow = (lane < K) ? rowi[q * K + lane] : -1;
            // Warp-uniform trip count (the shuffles below need all 32 lanes);
            // accesses past the row end are predicated off.
            for (int c0 = 0; c0 < n16; c0 += 32 * U) {
                const int c = c0 + lane;
                uint4 v[U];
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (c + 32 * u < n16) v[u] = ld_stream(src + c + 32 * u);
                for (int k = 0; k < K; ++k) {
                    const int r = __shfl_sync(kFull, myrow, k);
                    if (r < 0) continue;
                    uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)r * H);
#pragma unroll
                    for (int u = 0; u < U; ++u)
                        if (c + 32 * u < n16) st_vec(dst + c + 32 * u, v[u]);
                }
            }
        }
        __syncthreads();
    }
    warp_status_or(status, bad);

    // ---- pad rows [off[e] + c_e, off[e+1]) and the tail [N_pad, N_cap) ----
    int* padstart = base;  // [E+1] exclusive prefix of pad rows per expert
    for (int e = tid; e < E; e += kBlock) padstart[e] = (offsets[e + 1] - offsets[e]) - ecount[e];
    __syncthreads();
    const int P = block_exclusive_scan<MOE_MAX_E / kBlock>(padstart, E, scratch);
    if (tid == 0) padstart[E] = P;
    __syncthreads();

    const int gwarp = blockIdx.x * kWarps + warp;
    const int nwarps = gridDim.x * kWarps;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    for (int q = gwarp; q < P; q += nwarps) {
        const int e = upper_index(padstart, E + 1, q);
        const int64_t row = (int64_t)offsets[e] + ecount[e] + (q - padstart[e]);
        if (row < 0 || row >= N_cap) continue;
        if (lane == 0) r2f[row] = -1;
        if (zero_pad) {
            uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)row * H);
            for (int c = lane; c < n16; c += 32) st_vec(dst + c, zero);
        }
    }
    const int64_t gtid = (int64_t)blockIdx.x * kBlock + tid;
    const int64_t tail0 = N_pad > 0 ? N_pad : 0;
    for (int64_t row = tail0 + gtid; row < N_cap; row += (int64_t)gridDim.x * kBlock) r2f[row] = -1;
}

cudaError_t launch_permute(const uint16_t* x, const int64_t* topk_idx, int T, int K, int E, int H,
                           const int32_t* expert_offsets, const void* workspace, int zero_pad,
                           int64_t N_cap, uint16_t* x_perm, int32_t* row_to_flat,
                           int32_t* flat_to_row, int32_t* status, cudaStream_t stream) {
    // The tile geometry and the workspace parts are read from the header on
    // the device, so R is not an argument.  Host-side bounds: every tile holds
    // at least one token (n_tiles <= T), and the cap TT <= T/R only shrinks
    // TT as R grows, so TT(R = 1) bounds the shared-memory tile buffers.
    const int sms = sm_count_current_device();
    int grid = sms * 4;
    if (grid > T) grid = T;
    if (grid < 1) grid = 1;
    const int TTmax = layout_geometry(T, K, 1).TT;
    const size_t smem = sizeof(int) * ((size_t)E + 1 + 2 * (size_t)TTmax * K);
    const char* ws = static_cast<const char*>(workspace);
    if (H >= 4096)
        permute_kernel<4><<<grid, kBlock, smem, stream>>>(x, topk_idx, T, K, E, H, expert_offsets,
                                                          ws, zero_pad, N_cap, x_perm, row_to_flat,
                                                          flat_to_row, status);
    else
        permute_kernel<8><<<grid, kBlock, smem, stream>>>(x, topk_idx, T, K, E, H, expert_offsets,
                                                          ws, zero_pad, N_cap, x_perm, row_to_flat,
                                                          flat_to_row, status);
    return cudaGetLastError();
}

}  // namespace moe
