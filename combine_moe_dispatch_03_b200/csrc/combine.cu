// combine.cu -- fused_weighted_restore and its backward.
//
// Source: DeepSpeed PR "AutoEP: support combine_impl=fused_weighted_sum with
// AutoEP+AutoTP folding" (Change: flat index token*top_k+slot, router-dtype
// weights as [tokens, top_k], coverage RuntimeError; Problem: the default
// restore rounds every product and add to the activation dtype, the fused one
// accumulates in FP32; Tests / Benchmark: row and score gradients), and the
// DeepEP issue "Does Deepep's Dispatch/Combine Support Autograd Like PyTorch's
// all_to_all?" (combine; dispatch backward is a combine with unit weights;
// combine backward is a dispatch).
//
// Forward, per token t and element h (FP32, slot order fixed, one rounding):
//     acc = 0;  acc = fmaf(w[t,k], y[row(t,k), h], acc)  for k = 0..K-1
//     out[t, h] = bf16_rn(acc)
// Backward, with g = grad_out:
//     grad_rows[row(t,k)] = bf16_rn(fp32(w[t,k] * g[t]))
//     grad_w[t,k] = sum_h g[t,h] * y[row(t,k), h]   (exact fp32 products, fp64 sum)
//
// The gathers are what cost: K scattered rows per token.  DRAM serves them
// best as long contiguous runs, so for K <= 8 the kernels are "slot-major":
// a warp walks the slots in order and fetches a contiguous 1-4 KB chunk of
// each slot's row, keeping D chunks in flight (a ring in registers), instead
// of fetching a 512-byte sliver of all K rows at once.  For K > 8 a generic
// warp-per-token kernel serves any K.
#include "common.cuh"
#include "internal.h"

namespace moe {

// Row element types.  A 16-byte vector holds kPer elements; unpack widens
// them to fp32 exactly, pack rounds fp32 values to the row type (RNE for
// bf16, nothing for fp32), prod is the exact product of a gradient and a row
// element in fp64 (bf16 x bf16 is exact already in fp32; fp32 x fp32 is exact
// in fp64).  The fp32 rows are the activation-dtype-fp32 case of the
// DeepSpeed folding PR's Tests ("fp32 and bf16 rows").
struct RowBf16 {
    static constexpr int kPer = 8;
    __device__ __forceinline__ static void unpack(const uint4& v, float (&f)[8]) { unpack8(v, f); }
    __device__ __forceinline__ static uint4 pack(const float (&f)[8]) { return pack8(f); }
    __device__ __forceinline__ static double prod(float g, float y) { return (double)__fmul_rn(g, y); }
};
struct RowF32 {
    static constexpr int kPer = 4;
    __device__ __forceinline__ static void unpack(const uint4& v, float (&f)[4]) {
        f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
    }
    __device__ __forceinline__ static uint4 pack(const float (&f)[4]) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                          __float_as_uint(f[3]));
    }
    __device__ __forceinline__ static double prod(float g, float y) { return (double)g * (double)y; }
};

// ------------------------------------------------- forward, any K ---
// One warp per token; for each column chunk of 32 x U vectors the slots are
// visited in order (any K up to MOE_MAX_K).
template <typename Tr, int U, bool VALIDATE>
__global__ void __launch_bounds__(kBlock)
combine_kernel(const uint4* __restrict__ rows, int64_t N_cap, const int32_t* __restrict__ r2f,
               const int32_t* __restrict__ f2r, const void* __restrict__ w, int wdtype, int T,
               int K, int n16, uint4* __restrict__ out, int32_t* __restrict__ status) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    pdl_wait();
    pdl_trigger();
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    int bad = 0;

    for (int t = blockIdx.x * kWarps + warp; t < T; t += gridDim.x * kWarps) {
        int myrow = -1;
        float myw = 0.f;
        if (lane < K) {
            const int64_t f = (int64_t)t * K + lane;
            int r = f2r[f];
            if (r < 0 || (int64_t)r >= N_cap) {
                bad |= MOE_ST_ROW_OOR;
                r = -1;
            } else {
                myw = w ? load_weight(w, wdtype, f) : 1.f;
                if (VALIDATE && r2f[r] != (int32_t)f) bad |= MOE_ST_COVERAGE;
            }
            myrow = r;
        }
        uint4* dst = out + (size_t)t * n16;
        // Warp-uniform trip count: the shuffles inside need all 32 lanes.
        for (int c0 = 0; c0 < n16; c0 += 32 * U) {
            const int c = c0 + lane;
            float acc[U][Tr::kPer];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int i = 0; i < Tr::kPer; ++i) acc[u][i] = 0.f;
            for (int k = 0; k < K; ++k) {
                const int r = __shfl_sync(kFull, myrow, k);
                const float wv = __shfl_sync(kFull, myw, k);
                if (r < 0) continue;
                const uint4* src = rows + (size_t)r * n16;
                uint4 v[U];
#pragma unroll
                for (int u = 0; u < U; ++u)
                    v[u] = (c + 32 * u < n16) ? ld_stream(src + c + 32 * u) : zero;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    float y[Tr::kPer];
                    Tr::unpack(v[u], y);
#pragma unroll
                    for (int i = 0; i < Tr::kPer; ++i) acc[u][i] = __fmaf_rn(wv, y[i], acc[u][i]);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (c + 32 * u < n16) st_vec(dst + c + 32 * u, Tr::pack(acc[u]));
        }
    }

    if (VALIDATE) {
        // Row side of the bijection: every row that claims a (token, slot)
        // must be the row that (token, slot) points to.
        const int64_t A = (int64_t)T * K;
        const int64_t stride = (int64_t)gridDim.x * kBlock;
        for (int64_t row = (int64_t)blockIdx.x * kBlock + threadIdx.x; row < N_cap; row += stride) {
            const int32_t f = r2f[row];
            if (f < 0) continue;
            if ((int64_t)f >= A || (int64_t)f2r[f] != row) bad |= MOE_ST_COVERAGE;
        }
    }
    warp_status_or(status, bad);
}

// ------------------------------------------------- forward, slot-major ---
//
// One warp per (token, column chunk) item; a chunk is 32 lanes x U 16-byte
// vectors (2 KB for U = 4).  The warp walks the slots k = 0..K-1 in order
// and, for each, loads that slot's row chunk -- a contiguous run, the access
// pattern DRAM serves best -- keeping D row chunks in flight (a ring), and
// applies acc = fmaf(w_k, y, acc) as each chunk lands.  Same arithmetic and
// order as combine_kernel.
#ifndef MOE_COMBINE_U
#define MOE_COMBINE_U 2
#endif
#ifndef MOE_COMBINE_D
#define MOE_COMBINE_D 4
#endif

// Where a slot's row lives.  A Slot names one slot's row: LocalRows, one
// expert-grouped buffer, names it by its row index (from flat_to_row; -1
// for a skipped slot); RankRows, the buffer of the rank that owns the slot's
// expert (a table of R buffers, peer addresses across GPUs; plain loads),
// names it by a pointer to the row (nullptr for a skipped slot).
struct LocalRows {
    const uint4* rows;
    const int32_t* r2f;
    using Slot = int;
    static constexpr bool kRowSweep = true;
    // Coverage: the row claims this (token, slot).
    __device__ __forceinline__ bool check(int64_t f, int r) const { return r2f[r] == (int32_t)f; }
    __device__ __forceinline__ static Slot none() { return -1; }
    __device__ __forceinline__ bool expert_ok(int64_t) const { return true; }
    __device__ __forceinline__ Slot slot(int64_t, int r, int) const { return r; }
    __device__ __forceinline__ static bool valid(Slot s) { return s >= 0; }
    __device__ __forceinline__ const uint4* ptr(Slot s, int n16) const {
        return rows + (size_t)(s < 0 ? 0 : s) * n16;
    }
    __device__ __forceinline__ static Slot shfl(Slot s, int k) { return __shfl_sync(kFull, s, k); }
};
struct RankRows {
    const uint4* const* rows;
    const int64_t* topk;
    const int32_t* const* claims;   // per rank, the claim of every row
    int E, El, rank;
    using Slot = const uint4*;
    // Coverage can only be checked from the slot side: the row in its owner's
    // buffer must be claimed by this rank's (token, slot).
    static constexpr bool kRowSweep = false;
    __device__ __forceinline__ bool check(int64_t f, int r) const {
        return claims[topk[f] / El][r] == claim_code(rank, f);
    }
    __device__ __forceinline__ static Slot none() { return nullptr; }
    __device__ __forceinline__ bool expert_ok(int64_t f) const {
        const int64_t e = topk[f];
        return e >= 0 && e < E;
    }
    __device__ __forceinline__ Slot slot(int64_t f, int r, int n16) const {
        return rows[topk[f] / El] + (size_t)r * n16;
    }
    __device__ __forceinline__ static bool valid(Slot s) { return s != nullptr; }
    __device__ __forceinline__ const uint4* ptr(Slot s, int) const { return s; }
    __device__ __forceinline__ static Slot shfl(Slot s, int k) {
        return reinterpret_cast<Slot>(
            __shfl_sync(kFull, reinterpret_cast<unsigned long long>(s), k));
    }
};

template <typename Tr, int KT, int U, int D, bool VALIDATE, typename Src>
__global__ void __launch_bounds__(kBlock)
combine_slots_kernel(Src src_rows, int64_t N_cap, const int32_t* __restrict__ r2f,
                     const int32_t* __restrict__ f2r, const void* __restrict__ w, int wdtype,
                     int T, int n16, uint4* __restrict__ out, int32_t* __restrict__ status) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    pdl_wait();
    pdl_trigger();
    const int chunks = (n16 + 32 * U - 1) / (32 * U);
    const int64_t n_items = (int64_t)T * chunks;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    int bad = 0;

    for (int64_t item = (int64_t)blockIdx.x * kWarps + warp; item < n_items;
         item += (int64_t)gridDim.x * kWarps) {
        const int64_t t = item / chunks;
        const int c = (int)(item - t * chunks);
        // Lane k < KT resolves slot k: its row and its weight.
        typename Src::Slot myrow = Src::none();
        float myw = 0.f;
        if (lane < KT) {
            const int64_t f = t * KT + lane;
            const int r = f2r[f];
            if (r < 0 || (int64_t)r >= N_cap || !src_rows.expert_ok(f)) {
                if (c == 0) bad |= MOE_ST_ROW_OOR;
            } else {
                myw = w ? load_weight(w, wdtype, f) : 1.f;
                if (VALIDATE && c == 0 && !src_rows.check(f, r)) bad |= MOE_ST_COVERAGE;
                myrow = src_rows.slot(f, r, n16);
            }
        }
        typename Src::Slot rk[KT];
        float wk[KT];
#pragma unroll
        for (int k = 0; k < KT; ++k) {
            rk[k] = Src::shfl(myrow, k);
            wk[k] = __shfl_sync(kFull, myw, k);
        }
        const int v0 = c * 32 * U + lane;
        uint4 ring[D][U];
#pragma unroll
        for (int k = 0; k < D && k < KT; ++k) {
            const uint4* src = src_rows.ptr(rk[k], n16);
#pragma unroll
            for (int u = 0; u < U; ++u)
                ring[k][u] = (Src::valid(rk[k]) && v0 + 32 * u < n16) ? ld_stream(src + v0 + 32 * u) : zero;
        }
        float acc[U][Tr::kPer];
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int i = 0; i < Tr::kPer; ++i) acc[u][i] = 0.f;
#pragma unroll
        for (int k = 0; k < KT; ++k) {
            const int slot = k % D;
            if (Src::valid(rk[k])) {
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    float y[Tr::kPer];
                    Tr::unpack(ring[slot][u], y);
#pragma unroll
                    for (int i = 0; i < Tr::kPer; ++i) acc[u][i] = __fmaf_rn(wk[k], y[i], acc[u][i]);
                }
            }
            if (k + D < KT) {
                const int kn = k + D;
                const uint4* src = src_rows.ptr(rk[kn], n16);
#pragma unroll
                for (int u = 0; u < U; ++u)
                    ring[slot][u] = (Src::valid(rk[kn]) && v0 + 32 * u < n16) ? ld_stream(src + v0 + 32 * u) : zero;
            }
        }
        uint4* dst = out + (size_t)t * n16;
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (v0 + 32 * u < n16) st_vec(dst + v0 + 32 * u, Tr::pack(acc[u]));
    }

    if constexpr (VALIDATE && Src::kRowSweep) {
        const int64_t A = (int64_t)T * KT;
        const int64_t stride = (int64_t)gridDim.x * kBlock;
        for (int64_t row = (int64_t)blockIdx.x * kBlock + threadIdx.x; row < N_cap; row += stride) {
            const int32_t f = r2f[row];
            if (f < 0) continue;
            if ((int64_t)f >= A || (int64_t)f2r[f] != row) bad |= MOE_ST_COVERAGE;
        }
    }
    warp_status_or(status, bad);
}

// ------------------------------------------------ backward, any K ---
// One warp per token, one slot at a time over the whole row (g is re-read
// per slot from cache); the weight gradient is reduced per slot.
template <typename Tr>
__global__ void __launch_bounds__(kBlock)
combine_bwd_kernel(const uint4* __restrict__ g, const uint4* __restrict__ rows,
                   int64_t N_cap, const int32_t* __restrict__ r2f,
                   const int32_t* __restrict__ f2r, const void* __restrict__ w, int wdtype, int T,
                   int K, int n16, const int32_t* __restrict__ offsets, int E, int zero_pad,
                   uint4* __restrict__ grad_rows, void* __restrict__ grad_w,
                   int32_t* __restrict__ status) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    pdl_wait();
    pdl_trigger();
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    int bad = 0;

    for (int t = blockIdx.x * kWarps + warp; t < T; t += gridDim.x * kWarps) {
        int myrow = -1;
        float myw = 0.f;
        if (lane < K) {
            const int64_t f = (int64_t)t * K + lane;
            int r = f2r[f];
            if (r < 0 || (int64_t)r >= N_cap) {
                bad |= MOE_ST_ROW_OOR;
                r = -1;
            } else {
                myw = load_weight(w, wdtype, f);
            }
            myrow = r;
        }
        const uint4* gsrc = g + (size_t)t * n16;
        for (int k = 0; k < K; ++k) {
            const int r = __shfl_sync(kFull, myrow, k);
            const float wv = __shfl_sync(kFull, myw, k);
            double dk = 0.0;
            if (r >= 0) {
                const uint4* src = rows + (size_t)r * n16;
                uint4* dst = grad_rows + (size_t)r * n16;
                for (int c = lane; c < n16; c += 32) {
                    float gf[Tr::kPer], yf[Tr::kPer], o[Tr::kPer];
                    Tr::unpack(gsrc[c], gf);
                    Tr::unpack(ld_stream(src + c), yf);
                    double part = 0.0;
#pragma unroll
                    for (int i = 0; i < Tr::kPer; ++i) {
                        part += Tr::prod(gf[i], yf[i]);   // exact
                        o[i] = __fmul_rn(wv, gf[i]);
                    }
                    dk += part;
                    st_vec(dst + c, Tr::pack(o));
                }
            }
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) dk += __shfl_xor_sync(kFull, dk, d);
            if (grad_w && lane == 0) {
                const int64_t f = (int64_t)t * K + k;
                if (wdtype == MOE_DTYPE_F32) {
                    static_cast<float*>(grad_w)[f] = __double2float_rn(dk);
                } else {
                    __nv_bfloat16 b = __double2bfloat16(dk);
                    static_cast<uint16_t*>(grad_w)[f] = *reinterpret_cast<uint16_t*>(&b);
                }
            }
        }
    }

    if (zero_pad) {
        // Pad rows below offsets[E]: 32 rows per warp step, flagged by a
        // coalesced read of row_to_flat, zeroed with full-row vector stores.
        const int64_t N_pad = offsets[E];
        const int64_t limit = N_pad < N_cap ? N_pad : N_cap;
        const int64_t wstride = (int64_t)gridDim.x * kWarps * 32;
        for (int64_t base = ((int64_t)blockIdx.x * kWarps + warp) * 32; base < limit; base += wstride) {
            const int64_t row = base + lane;
            const bool pad = row < limit && r2f[row] < 0;
            unsigned m = __ballot_sync(kFull, pad);
            while (m) {
                const int b = __ffs(m) - 1;
                m &= m - 1;
                uint4* dst = grad_rows + (size_t)(base + b) * n16;
                for (int c = lane; c < n16; c += 32) st_vec(dst + c, zero);
            }
        }
    }
    warp_status_or(status, bad);
}

// ------------------------------------------------ backward, slot-major ---
//
// One warp per token.  The row is walked in chunks of 32 lanes x U vectors;
// per chunk, g is loaded once, then the slots k = 0..K-1 are visited in
// order with D row chunks of y in flight (a ring): the dot product with g
// accumulates in fp64 per slot (registers, across chunks), and the slot's
// gradient chunk bf16_rn(w_k * g) is stored as a contiguous run.
#ifndef MOE_BWD_MIN_BLOCKS
#define MOE_BWD_MIN_BLOCKS 2
#endif

template <typename Tr, int KT, int U, int D>
__global__ void __launch_bounds__(kBlock, MOE_BWD_MIN_BLOCKS)
combine_bwd_slots_kernel(const uint4* __restrict__ g, const uint4* __restrict__ rows,
                         int64_t N_cap, const int32_t* __restrict__ r2f,
                         const int32_t* __restrict__ f2r, const void* __restrict__ w, int wdtype,
                         int T, int n16, const int32_t* __restrict__ offsets, int E, int zero_pad,
                         uint4* __restrict__ grad_rows, void* __restrict__ grad_w,
                         int32_t* __restrict__ status) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    pdl_wait();
    pdl_trigger();
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    int bad = 0;

    for (int t = blockIdx.x * kWarps + warp; t < T; t += gridDim.x * kWarps) {
        int myrow = -1;
        float myw = 0.f;
        if (lane < KT) {
            const int64_t f = (int64_t)t * KT + lane;
            int r = f2r[f];
            if (r < 0 || (int64_t)r >= N_cap) {
                bad |= MOE_ST_ROW_OOR;
                r = -1;
            } else {
                myw = load_weight(w, wdtype, f);
            }
            myrow = r;
        }
        int rk[KT];
        float wk[KT];
        double dot[KT];
#pragma unroll
        for (int k = 0; k < KT; ++k) {
            rk[k] = __shfl_sync(kFull, myrow, k);
            wk[k] = __shfl_sync(kFull, myw, k);
            dot[k] = 0.0;
        }
        const uint4* gsrc = g + (size_t)t * n16;
        for (int c0 = 0; c0 < n16; c0 += 32 * U) {
            const int v0 = c0 + lane;
            uint4 gv[U];
#pragma unroll
            for (int u = 0; u < U; ++u) gv[u] = (v0 + 32 * u < n16) ? ld_stream(gsrc + v0 + 32 * u) : zero;
            uint4 ring[D][U];
#pragma unroll
            for (int k = 0; k < D && k < KT; ++k) {
                const uint4* src = rows + (size_t)(rk[k] < 0 ? 0 : rk[k]) * n16;
#pragma unroll
                for (int u = 0; u < U; ++u)
                    ring[k][u] = (rk[k] >= 0 && v0 + 32 * u < n16) ? ld_stream(src + v0 + 32 * u) : zero;
            }
#pragma unroll
            for (int k = 0; k < KT; ++k) {
                const int slot = k % D;
                if (rk[k] >= 0) {
                    uint4* dst = grad_rows + (size_t)rk[k] * n16;
                    double part = 0.0;
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        if (v0 + 32 * u >= n16) continue;
                        float gf[Tr::kPer], yf[Tr::kPer], o[Tr::kPer];
                        Tr::unpack(gv[u], gf);
                        Tr::unpack(ring[slot][u], yf);
#pragma unroll
                        for (int i = 0; i < Tr::kPer; ++i) {
                            part += Tr::prod(gf[i], yf[i]);   // exact
                            o[i] = __fmul_rn(wk[k], gf[i]);
                        }
                        st_vec(dst + v0 + 32 * u, Tr::pack(o));
                    }
                    dot[k] += part;
                }
                if (k + D < KT) {
                    const int kn = k + D;
                    const uint4* src = rows + (size_t)(rk[kn] < 0 ? 0 : rk[kn]) * n16;
#pragma unroll
                    for (int u = 0; u < U; ++u)
                        ring[slot][u] = (rk[kn] >= 0 && v0 + 32 * u < n16) ? ld_stream(src + v0 + 32 * u) : zero;
                }
            }
        }
        if (grad_w) {
#pragma unroll
            for (int k = 0; k < KT; ++k) {
                double v = dot[k];
#pragma unroll
                for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(kFull, v, d);
                if (lane == k) {
                    const int64_t f = (int64_t)t * KT + k;
                    if (wdtype == MOE_DTYPE_F32) {
                        static_cast<float*>(grad_w)[f] = __double2float_rn(v);
                    } else {
                        __nv_bfloat16 b = __double2bfloat16(v);
                        static_cast<uint16_t*>(grad_w)[f] = *reinterpret_cast<uint16_t*>(&b);
                    }
                }
            }
        }
    }

    if (zero_pad) {
        const int64_t N_pad = offsets[E];
        const int64_t limit = N_pad < N_cap ? N_pad : N_cap;
        const int64_t wstride = (int64_t)gridDim.x * kWarps * 32;
        for (int64_t base = ((int64_t)blockIdx.x * kWarps + warp) * 32; base < limit; base += wstride) {
            const int64_t row = base + lane;
            const bool pad = row < limit && r2f[row] < 0;
            unsigned m = __ballot_sync(kFull, pad);
            while (m) {
                const int b = __ffs(m) - 1;
                m &= m - 1;
                uint4* dst = grad_rows + (size_t)(base + b) * n16;
                for (int c = lane; c < n16; c += 32) st_vec(dst + c, zero);
            }
        }
    }
    warp_status_or(status, bad);
}

// ------------------------------------------------------------ launchers ---

template <typename Tr, bool V>
static void launch_combine_t(int K, int grid, cudaStream_t st, const uint4* rows, int64_t N_cap,
                             const int32_t* r2f, const int32_t* f2r, const void* w, int wd, int T,
                             int n16, uint4* out, int32_t* status) {
    launch_pdl(combine_kernel<Tr, 2, V>, dim3(grid), dim3(kBlock), 0, st, rows, N_cap, r2f, f2r, w,
               wd, T, K, n16, out, status);
}

// Enough warps for one token each (up to 8 resident CTAs per SM), and, when a
// row sweep follows, enough threads to cover the rows.
#ifndef MOE_BWD_GRID_PER_SM
#define MOE_BWD_GRID_PER_SM 8
#endif
static int grid_tokens_and_rows(int T, int64_t N_cap, bool sweep_rows, int per_sm = 8) {
    const int cap = sm_count_current_device() * per_sm;
    int64_t want = (T + kWarps - 1) / kWarps;
    if (sweep_rows) {
        const int64_t rw = (N_cap + kBlock - 1) / kBlock;
        if (rw > want) want = rw;
    }
    if (want > cap) want = cap;
    return want < 1 ? 1 : (int)want;
}

#define MOE_SLOTS_ARGS src, N_cap, r2f, f2r, w, wd, T, n16, out, status

template <typename Tr, bool V, typename Src>
static void launch_slots_t(int K, int grid, cudaStream_t st, Src src, int64_t N_cap,
                           const int32_t* r2f, const int32_t* f2r, const void* w, int wd, int T,
                           int n16, uint4* out, int32_t* status) {
    constexpr int U = MOE_COMBINE_U, D = MOE_COMBINE_D;
    // Small K: wider chunks keep as many vectors in flight per lane.
    switch (K) {
        case 1: launch_pdl(combine_slots_kernel<Tr, 1, 4 * U, 1, V, Src>, dim3(grid), dim3(kBlock), 0, st, MOE_SLOTS_ARGS); break;
        case 2: launch_pdl(combine_slots_kernel<Tr, 2, 2 * U, 2, V, Src>, dim3(grid), dim3(kBlock), 0, st, MOE_SLOTS_ARGS); break;
        case 3: launch_pdl(combine_slots_kernel<Tr, 3, U, (D < 3 ? D : 3), V, Src>, dim3(grid), dim3(kBlock), 0, st, MOE_SLOTS_ARGS); break;
        case 4: launch_pdl(combine_slots_kernel<Tr, 4, U, D, V, Src>, dim3(grid), dim3(kBlock), 0, st, MOE_SLOTS_ARGS); break;
        case 5: launch_pdl(combine_slots_kernel<Tr, 5, U, D, V, Src>, dim3(grid), dim3(kBlock), 0, st, MOE_SLOTS_ARGS); break;
        case 6: launch_pdl(combine_slots_kernel<Tr, 6, U, D, V, Src>, dim3(grid), dim3(kBlock), 0, st, MOE_SLOTS_ARGS); break;
        case 7: launch_pdl(combine_slots_kernel<Tr, 7, U, D, V, Src>, dim3(grid), dim3(kBlock), 0, st, MOE_SLOTS_ARGS); break;
        default: launch_pdl(combine_slots_kernel<Tr, 8, U, D, V, Src>, dim3(grid), dim3(kBlock), 0, st, MOE_SLOTS_ARGS); break;
    }
}

// Grid of the slot-major kernels: one warp per (token, chunk) item, up to
// MOE_COMBINE_GRID_PER_SM resident CTAs per SM, and with validation enough
// threads to sweep the rows.
#ifndef MOE_COMBINE_GRID_PER_SM
#define MOE_COMBINE_GRID_PER_SM 8
#endif
static int slots_grid(int T, int K, int n16, int64_t N_cap, bool validate) {
    const int u = K == 1 ? 4 * MOE_COMBINE_U : (K == 2 ? 2 * MOE_COMBINE_U : MOE_COMBINE_U);
    const int chunks = (n16 + 32 * u - 1) / (32 * u);
    const int64_t items = (int64_t)T * chunks;
    const int cap = sm_count_current_device() * MOE_COMBINE_GRID_PER_SM;
    int64_t want = (items + kWarps - 1) / kWarps;
    if (validate) {
        const int64_t rw = (N_cap + kBlock - 1) / kBlock;
        if (rw > want) want = rw;
    }
    return (int)(want > cap ? cap : (want < 1 ? 1 : want));
}

template <typename Tr>
static cudaError_t launch_combine_rows(const uint4* rows, int64_t N_cap, const int32_t* r2f,
                                       const int32_t* f2r, const void* w, int wd, int T, int K,
                                       int n16, int validate, uint4* out, int32_t* status,
                                       cudaStream_t stream) {
    if (K <= 8) {
        const int grid = slots_grid(T, K, n16, N_cap, validate != 0);
        const LocalRows src{rows, r2f};
        if (validate)
            launch_slots_t<Tr, true>(K, grid, stream, src, N_cap, r2f, f2r, w, wd, T, n16, out,
                                     status);
        else
            launch_slots_t<Tr, false>(K, grid, stream, src, N_cap, r2f, f2r, w, wd, T, n16, out,
                                      status);
        return cudaGetLastError();
    }
    const int grid = grid_tokens_and_rows(T, N_cap, validate != 0);
    if (validate)
        launch_combine_t<Tr, true>(K, grid, stream, rows, N_cap, r2f, f2r, w, wd, T, n16, out,
                                   status);
    else
        launch_combine_t<Tr, false>(K, grid, stream, rows, N_cap, r2f, f2r, w, wd, T, n16, out,
                                    status);
    return cudaGetLastError();
}

// The slot-major restore with every slot's row read from the buffer of its
// expert's rank (K <= 8); the generic kernel in ranks.cu serves larger K.
cudaError_t launch_combine_slots_from_ranks(const uint16_t* const* rows,
                                            const int32_t* const* claims, int R, int rank,
                                            int64_t N_cap, const int32_t* flat_to_row,
                                            const int64_t* topk_idx, int E, const void* weights,
                                            int weight_dtype, int T, int K, int H, uint16_t* out,
                                            int32_t* status, cudaStream_t stream) {
    const int n16 = H / 8;
    const RankRows src{reinterpret_cast<const uint4* const*>(rows), topk_idx, claims, E, E / R,
                       rank};
    const int grid = slots_grid(T, K, n16, N_cap, false);
    if (claims)
        launch_slots_t<RowBf16, true>(K, grid, stream, src, N_cap, nullptr, flat_to_row, weights,
                                      weight_dtype, T, n16, reinterpret_cast<uint4*>(out), status);
    else
        launch_slots_t<RowBf16, false>(K, grid, stream, src, N_cap, nullptr, flat_to_row, weights,
                                       weight_dtype, T, n16, reinterpret_cast<uint4*>(out), status);
    return cudaGetLastError();
}

cudaError_t launch_combine(const uint16_t* rows, int64_t N_cap, const int32_t* row_to_flat,
                           const int32_t* flat_to_row, const void* weights, int weight_dtype,
                           int T, int K, int H, int validate, uint16_t* out, int32_t* status,
                           cudaStream_t stream) {
    return launch_combine_rows<RowBf16>(reinterpret_cast<const uint4*>(rows), N_cap, row_to_flat,
                                        flat_to_row, weights, weight_dtype, T, K, H / 8, validate,
                                        reinterpret_cast<uint4*>(out), status, stream);
}

cudaError_t launch_combine_f32(const float* rows, int64_t N_cap, const int32_t* row_to_flat,
                               const int32_t* flat_to_row, const void* weights, int weight_dtype,
                               int T, int K, int H, int validate, float* out, int32_t* status,
                               cudaStream_t stream) {
    return launch_combine_rows<RowF32>(reinterpret_cast<const uint4*>(rows), N_cap, row_to_flat,
                                       flat_to_row, weights, weight_dtype, T, K, H / 4, validate,
                                       reinterpret_cast<uint4*>(out), status, stream);
}

#define MOE_BWD_SLOT_ARGS                                                                      \
    g, rows, N_cap, r2f, f2r, w, wd, T, n16, offsets, E, zero_pad, grad_rows, grad_w, status

template <typename Tr>
static cudaError_t launch_backward_rows(const uint4* g, const uint4* rows, int64_t N_cap,
                                        const int32_t* r2f, const int32_t* f2r, const void* w,
                                        int wd, int T, int K, int n16, const int32_t* offsets,
                                        int E, int zero_pad, uint4* grad_rows, void* grad_w,
                                        int32_t* status, cudaStream_t stream) {
    const int grid = grid_tokens_and_rows(T, N_cap, zero_pad != 0, MOE_BWD_GRID_PER_SM);
#ifndef MOE_BWD_U
#define MOE_BWD_U MOE_COMBINE_U
#endif
#ifndef MOE_BWD_D
#define MOE_BWD_D MOE_COMBINE_D
#endif
    constexpr int U = MOE_BWD_U, D = MOE_BWD_D;
    switch (K) {
        case 1: launch_pdl(combine_bwd_slots_kernel<Tr, 1, 4 * U, 1>, dim3(grid), dim3(kBlock), 0, stream, MOE_BWD_SLOT_ARGS); break;
        case 2: launch_pdl(combine_bwd_slots_kernel<Tr, 2, 2 * U, 2>, dim3(grid), dim3(kBlock), 0, stream, MOE_BWD_SLOT_ARGS); break;
        case 3: launch_pdl(combine_bwd_slots_kernel<Tr, 3, U, (D < 3 ? D : 3)>, dim3(grid), dim3(kBlock), 0, stream, MOE_BWD_SLOT_ARGS); break;
        case 4: launch_pdl(combine_bwd_slots_kernel<Tr, 4, U, D>, dim3(grid), dim3(kBlock), 0, stream, MOE_BWD_SLOT_ARGS); break;
        case 5: launch_pdl(combine_bwd_slots_kernel<Tr, 5, U, D>, dim3(grid), dim3(kBlock), 0, stream, MOE_BWD_SLOT_ARGS); break;
        case 6: launch_pdl(combine_bwd_slots_kernel<Tr, 6, U, D>, dim3(grid), dim3(kBlock), 0, stream, MOE_BWD_SLOT_ARGS); break;
        case 7: launch_pdl(combine_bwd_slots_kernel<Tr, 7, U, D>, dim3(grid), dim3(kBlock), 0, stream, MOE_BWD_SLOT_ARGS); break;
        case 8: launch_pdl(combine_bwd_slots_kernel<Tr, 8, U, D>, dim3(grid), dim3(kBlock), 0, stream, MOE_BWD_SLOT_ARGS); break;
        default:
            launch_pdl(combine_bwd_kernel<Tr>, dim3(grid), dim3(kBlock), 0, stream, g, rows, N_cap, r2f,
                       f2r, w, wd, T, K, n16, offsets, E, zero_pad, grad_rows, grad_w, status);
            break;
    }
    return cudaGetLastError();
}

cudaError_t launch_combine_backward(const uint16_t* grad_out, const uint16_t* rows, int64_t N_cap,
                                    const int32_t* row_to_flat, const int32_t* flat_to_row,
                                    const void* weights, int weight_dtype, int T, int K, int H,
                                    const int32_t* expert_offsets, int E, int zero_pad,
                                    uint16_t* grad_rows, void* grad_weights, int32_t* status,
                                    cudaStream_t stream) {
    return launch_backward_rows<RowBf16>(
        reinterpret_cast<const uint4*>(grad_out), reinterpret_cast<const uint4*>(rows), N_cap,
        row_to_flat, flat_to_row, weights, weight_dtype, T, K, H / 8, expert_offsets, E, zero_pad,
        reinterpret_cast<uint4*>(grad_rows), grad_weights, status, stream);
}

cudaError_t launch_combine_backward_f32(const float* grad_out, const float* rows, int64_t N_cap,
                                        const int32_t* row_to_flat, const int32_t* flat_to_row,
                                        const void* weights, int weight_dtype, int T, int K, int H,
                                        const int32_t* expert_offsets, int E, int zero_pad,
                                        float* grad_rows, void* grad_weights, int32_t* status,
                                        cudaStream_t stream) {
    return launch_backward_rows<RowF32>(
        reinterpret_cast<const uint4*>(grad_out), reinterpret_cast<const uint4*>(rows), N_cap,
        row_to_flat, flat_to_row, weights, weight_dtype, T, K, H / 4, expert_offsets, E, zero_pad,
        reinterpret_cast<uint4*>(grad_rows), grad_weights, status, stream);
}

}  // namespace moe
