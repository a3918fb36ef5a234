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
// One warp per token, grid-stride.  Lane k < K fetches slot k's row index and
// weight once; the row indices are then broadcast to registers, so for every
// 16-byte column chunk the warp issues the K gathers back to back (K*U
// vectors in flight per lane) before the fixed-order FMA chain.  Reads are
// coalesced 512-byte row segments; the output row is written once.
#include "common.cuh"
#include "internal.h"

namespace moe {

// ------------------------------------------------------------- forward ---

template <int KT, int U, bool VALIDATE>
__global__ void __launch_bounds__(kBlock)
combine_kernel(const uint16_t* __restrict__ rows, int64_t N_cap, const int32_t* __restrict__ r2f,
               const int32_t* __restrict__ f2r, const void* __restrict__ w, int wdtype, int T,
               int K, int H, uint16_t* __restrict__ out, int32_t* __restrict__ status) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int Kn = KT > 0 ? KT : K;
    const int n16 = H >> 3;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    int bad = 0;

    for (int t = blockIdx.x * kWarps + warp; t < T; t += gridDim.x * kWarps) {
        int myrow = -1;
        float myw = 0.f;
        if (lane < Kn) {
            const int64_t f = (int64_t)t * Kn + lane;
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
        uint4* dst = reinterpret_cast<uint4*>(out + (size_t)t * H);
        if constexpr (KT > 0) {
            int rk[KT];
            float wk[KT];
#pragma unroll
            for (int k = 0; k < KT; ++k) {
                rk[k] = __shfl_sync(kFull, myrow, k);
                wk[k] = __shfl_sync(kFull, myw, k);
            }
            for (int c = lane; c < n16; c += 32 * U) {
                uint4 v[KT][U];
#pragma unroll
                for (int k = 0; k < KT; ++k) {
                    const uint4* src = reinterpret_cast<const uint4*>(rows + (size_t)(rk[k] < 0 ? 0 : rk[k]) * H);
#pragma unroll
                    for (int u = 0; u < U; ++u)
                        v[k][u] = (rk[k] >= 0 && c + 32 * u < n16) ? ld_stream(src + c + 32 * u) : zero;
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (c + 32 * u >= n16) continue;
                    float acc[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
                    for (int k = 0; k < KT; ++k) {
                        float y[8];
                        unpack8(v[k][u], y);
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[i] = __fmaf_rn(wk[k], y[i], acc[i]);
                    }
                    st_vec(dst + c + 32 * u, pack8(acc));
                }
            }
        } else {
            // Warp-uniform trip count: the shuffles inside need all 32 lanes.
            for (int c0 = 0; c0 < n16; c0 += 32 * U) {
                const int c = c0 + lane;
                float acc[U][8];
#pragma unroll
                for (int u = 0; u < U; ++u)
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;
                for (int k = 0; k < Kn; ++k) {
                    const int r = __shfl_sync(kFull, myrow, k);
                    const float wv = __shfl_sync(kFull, myw, k);
                    if (r < 0) continue;
                    const uint4* src = reinterpret_cast<const uint4*>(rows + (size_t)r * H);
                    uint4 v[U];
#pragma unroll
                    for (int u = 0; u < U; ++u)
                        v[u] = (c + 32 * u < n16) ? ld_stream(src + c + 32 * u) : zero;
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
    }

    if (VALIDATE) {
        // Row side of the bijection: every row that claims a (token, slot)
        // must be the row that (token, slot) points to.
        const int64_t A = (int64_t)T * Kn;
        const int64_t stride = (int64_t)gridDim.x * kBlock;
        for (int64_t row = (int64_t)blockIdx.x * kBlock + threadIdx.x; row < N_cap; row += stride) {
            const int32_t f = r2f[row];
            if (f < 0) continue;
            if ((int64_t)f >= A || (int64_t)f2r[f] != row) bad |= MOE_ST_COVERAGE;
        }
    }
    warp_status_or(status, bad);
}

// ------------------------------------------------------------ backward ---

template <int KT, int U>
__global__ void __launch_bounds__(kBlock)
combine_bwd_kernel(const uint16_t* __restrict__ g, const uint16_t* __restrict__ rows,
                   int64_t N_cap, const int32_t* __restrict__ r2f,
                   const int32_t* __restrict__ f2r, const void* __restrict__ w, int wdtype, int T,
                   int K, int H, const int32_t* __restrict__ offsets, int E, int zero_pad,
                   uint16_t* __restrict__ grad_rows, void* __restrict__ grad_w,
                   int32_t* __restrict__ status) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n16 = H >> 3;
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
        const uint4* gsrc = reinterpret_cast<const uint4*>(g + (size_t)t * H);
        if constexpr (KT == 0) {
            // Any K: one slot at a time over the whole row (g is re-read per
            // slot from cache); the weight gradient is reduced per slot.
            for (int k = 0; k < K; ++k) {
                const int r = __shfl_sync(kFull, myrow, k);
                const float wv = __shfl_sync(kFull, myw, k);
                double dk = 0.0;
                if (r >= 0) {
                    const uint4* src = reinterpret_cast<const uint4*>(rows + (size_t)r * H);
                    uint4* dst = reinterpret_cast<uint4*>(grad_rows + (size_t)r * H);
                    for (int c = lane; c < n16; c += 32) {
                        float gf[8], yf[8], o[8];
                        unpack8(gsrc[c], gf);
                        unpack8(ld_stream(src + c), yf);
                        double part = 0.0;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            part += (double)__fmul_rn(gf[i], yf[i]);
                            o[i] = __fmul_rn(wv, gf[i]);
                        }
                        dk += part;
                        st_vec(dst + c, pack8(o));
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
            continue;
        } else {
        int rk[KT];
        float wk[KT];
        double dot[KT];
#pragma unroll
        for (int k = 0; k < KT; ++k) {
            rk[k] = __shfl_sync(kFull, myrow, k);
            wk[k] = __shfl_sync(kFull, myw, k);
            dot[k] = 0.0;
        }
        for (int c = lane; c < n16; c += 32 * U) {
            uint4 gv[U];
            uint4 yv[KT][U];
#pragma unroll
            for (int u = 0; u < U; ++u) gv[u] = (c + 32 * u < n16) ? ld_stream(gsrc + c + 32 * u) : zero;
#pragma unroll
            for (int k = 0; k < KT; ++k) {
                const uint4* src = reinterpret_cast<const uint4*>(rows + (size_t)(rk[k] < 0 ? 0 : rk[k]) * H);
#pragma unroll
                for (int u = 0; u < U; ++u)
                    yv[k][u] = (rk[k] >= 0 && c + 32 * u < n16) ? ld_stream(src + c + 32 * u) : zero;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (c + 32 * u >= n16) continue;
                float gf[8];
                unpack8(gv[u], gf);
#pragma unroll
                for (int k = 0; k < KT; ++k) {
                    if (rk[k] < 0) continue;
                    float yf[8], o[8];
                    unpack8(yv[k][u], yf);
                    double part = 0.0;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        part += (double)__fmul_rn(gf[i], yf[i]);   // exact: bf16 x bf16
                        o[i] = __fmul_rn(wk[k], gf[i]);
                    }
                    dot[k] += part;
                    uint4* dst = reinterpret_cast<uint4*>(grad_rows + (size_t)rk[k] * H);
                    st_vec(dst + c + 32 * u, pack8(o));
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
                uint4* dst = reinterpret_cast<uint4*>(grad_rows + (size_t)(base + b) * H);
                for (int c = lane; c < n16; c += 32) st_vec(dst + c, zero);
            }
        }
    }
    warp_status_or(status, bad);
}

// ------------------------------------------------------------ launchers ---

template <bool V>
static void launch_combine_t(int K, int grid, cudaStream_t st, const uint16_t* rows, int64_t N_cap,
                             const int32_t* r2f, const int32_t* f2r, const void* w, int wd, int T,
                             int H, uint16_t* out, int32_t* status) {
    switch (K) {
        case 1: combine_kernel<1, 8, V><<<grid, kBlock, 0, st>>>(rows, N_cap, r2f, f2r, w, wd, T, K, H, out, status); break;
        case 2: combine_kernel<2, 4, V><<<grid, kBlock, 0, st>>>(rows, N_cap, r2f, f2r, w, wd, T, K, H, out, status); break;
        case 4: combine_kernel<4, 2, V><<<grid, kBlock, 0, st>>>(rows, N_cap, r2f, f2r, w, wd, T, K, H, out, status); break;
        case 8: combine_kernel<8, 1, V><<<grid, kBlock, 0, st>>>(rows, N_cap, r2f, f2r, w, wd, T, K, H, out, status); break;
        default: combine_kernel<0, 2, V><<<grid, kBlock, 0, st>>>(rows, N_cap, r2f, f2r, w, wd, T, K, H, out, status); break;
    }
}

// Enough warps for one token each (up to 8 resident CTAs per SM), and, when a
// row sweep follows, enough threads to cover the rows.
static int grid_tokens_and_rows(int T, int64_t N_cap, bool sweep_rows) {
    const int cap = sm_count_current_device() * 8;
    int64_t want = (T + kWarps - 1) / kWarps;
    if (sweep_rows) {
        const int64_t rw = (N_cap + kBlock - 1) / kBlock;
        if (rw > want) want = rw;
    }
    if (want > cap) want = cap;
    return want < 1 ? 1 : (int)want;
}

cudaError_t launch_combine(const uint16_t* rows, int64_t N_cap, const int32_t* row_to_flat,
                           const int32_t* flat_to_row, const void* weights, int weight_dtype,
                           int T, int K, int H, int validate, uint16_t* out, int32_t* status,
                           cudaStream_t stream) {
    const int grid = grid_tokens_and_rows(T, N_cap, validate != 0);
    if (validate)
        launch_combine_t<true>(K, grid, stream, rows, N_cap, row_to_flat, flat_to_row, weights,
                               weight_dtype, T, H, out, status);
    else
        launch_combine_t<false>(K, grid, stream, rows, N_cap, row_to_flat, flat_to_row, weights,
                                weight_dtype, T, H, out, status);
    return cudaGetLastError();
}

#define MOE_BWD_ARGS                                                                           \
    grad_out, rows, N_cap, row_to_flat, flat_to_row, weights, weight_dtype, T, K, H,           \
        expert_offsets, E, zero_pad, grad_rows, grad_weights, status

cudaError_t launch_combine_backward(const uint16_t* grad_out, const uint16_t* rows, int64_t N_cap,
                                    const int32_t* row_to_flat, const int32_t* flat_to_row,
                                    const void* weights, int weight_dtype, int T, int K, int H,
                                    const int32_t* expert_offsets, int E, int zero_pad,
                                    uint16_t* grad_rows, void* grad_weights, int32_t* status,
                                    cudaStream_t stream) {
    const int grid = grid_tokens_and_rows(T, N_cap, zero_pad != 0);
    switch (K) {
        case 1: combine_bwd_kernel<1, 8><<<grid, kBlock, 0, stream>>>(MOE_BWD_ARGS); break;
        case 2: combine_bwd_kernel<2, 4><<<grid, kBlock, 0, stream>>>(MOE_BWD_ARGS); break;
        case 3: combine_bwd_kernel<3, 2><<<grid, kBlock, 0, stream>>>(MOE_BWD_ARGS); break;
        case 4: combine_bwd_kernel<4, 2><<<grid, kBlock, 0, stream>>>(MOE_BWD_ARGS); break;
        case 5: combine_bwd_kernel<5, 1><<<grid, kBlock, 0, stream>>>(MOE_BWD_ARGS); break;
        case 6: combine_bwd_kernel<6, 1><<<grid, kBlock, 0, stream>>>(MOE_BWD_ARGS); break;
        case 7: combine_bwd_kernel<7, 1><<<grid, kBlock, 0, stream>>>(MOE_BWD_ARGS); break;
        case 8: combine_bwd_kernel<8, 1><<<grid, kBlock, 0, stream>>>(MOE_BWD_ARGS); break;
        default: combine_bwd_kernel<0, 1><<<grid, kBlock, 0, stream>>>(MOE_BWD_ARGS); break;
    }
    return cudaGetLastError();
}

}  // namespace moe
