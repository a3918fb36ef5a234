// expert_scale.cu -- the seeded stand-in for the experts: y = bf16_rn(x * s_e)
// on every real row of expert e, zero on its pad rows.  It occupies the place
// of the grouped expert MLP (DeepSpeed AutoEP base PR, Design, step 5) so the
// dispatch -> experts -> combine chain can be checked end to end.
//
// One warp per row (grid-stride): the expert is found by binary search of the
// padded offsets in shared memory; a row is read once and written once with
// 16-byte vectors (pad rows are only written).
#include "common.cuh"
#include "internal.h"

namespace moe {

#ifndef MOE_SCALE_U
#define MOE_SCALE_U 4
#endif
#ifndef MOE_SCALE_GRID_PER_SM
#define MOE_SCALE_GRID_PER_SM 64
#endif

template <int U>
__global__ void __launch_bounds__(kBlock)
expert_scale_kernel(const uint16_t* __restrict__ rows, int64_t N_cap,
                    const int32_t* __restrict__ offsets, const int32_t* __restrict__ counts, int E,
                    int H, const float* __restrict__ scales, uint16_t* __restrict__ out,
                    int32_t* __restrict__ status) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    int* off = reinterpret_cast<int*>(smem_raw);  // [E+1]
    int* cnt = off + (E + 1);                      // [E]
    float* sc = reinterpret_cast<float*>(cnt + E); // [E]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();
    pdl_trigger();
    for (int e = tid; e <= E; e += kBlock) off[e] = offsets[e];
    for (int e = tid; e < E; e += kBlock) {
        cnt[e] = counts[e];
        sc[e] = scales[e];
    }
    __syncthreads();
    const int64_t N_pad = off[E];
    if (blockIdx.x == 0 && tid == 0 && N_pad > N_cap) atomicOr(status, MOE_ST_CAPACITY);
    const int64_t limit = N_pad < N_cap ? N_pad : N_cap;
    const int n16 = H >> 3;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);

    for (int64_t row = (int64_t)blockIdx.x * kWarps + warp; row < limit;
         row += (int64_t)gridDim.x * kWarps) {
        const int e = upper_index(off, E + 1, (int)row);
        const bool real = row < (int64_t)off[e] + cnt[e];
        const float s = sc[e];
        const uint4* src = reinterpret_cast<const uint4*>(rows + (size_t)row * H);
        uint4* dst = reinterpret_cast<uint4*>(out + (size_t)row * H);
        for (int c = lane; c < n16; c += 32 * U) {
            uint4 v[U];
            if (real) {
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (c + 32 * u < n16) v[u] = ld_stream(src + c + 32 * u);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (c + 32 * u >= n16) continue;
                uint4 o = zero;
                if (real) {
                    float f[8];
                    unpack8(v[u], f);
#pragma unroll
                    for (int i = 0; i < 8; ++i) f[i] = __fmul_rn(f[i], s);
                    o = pack8(f);
                }
                st_vec(dst + c + 32 * u, o);
            }
        }
    }
}

cudaError_t launch_expert_scale(const uint16_t* rows, int64_t N_cap, const int32_t* expert_offsets,
                                const int32_t* tokens_per_expert, int E, int H,
                                const float* scales, uint16_t* out, int32_t* status,
                                cudaStream_t stream) {
    const int sms = sm_count_current_device();
    int64_t want = (N_cap + kWarps - 1) / kWarps;
    int grid = sms * MOE_SCALE_GRID_PER_SM;
    if (want < grid) grid = (int)want;
    if (grid < 1) grid = 1;
    const size_t smem = sizeof(int) * (2 * (size_t)E + 1) + sizeof(float) * (size_t)E;
    return launch_pdl(expert_scale_kernel<MOE_SCALE_U>, dim3(grid), dim3(kBlock), smem, stream,
                      rows, N_cap, expert_offsets, tokens_per_expert, E, H, scales, out, status);
}

}  // namespace moe
