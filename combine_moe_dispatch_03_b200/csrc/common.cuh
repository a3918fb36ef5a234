// common.cuh -- device helpers shared by the dispatch/combine kernels.
//
// bf16 values travel as uint16 bit patterns packed eight to a 16-byte vector
// (uint4); every row is a whole number of vectors (H % 8 == 0), so every row
// copy is a sequence of aligned 16-byte loads and stores, coalesced across a
// warp (32 lanes x 16 B = 512 B per instruction).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "moe_dispatch.h"

namespace moe {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kBlock = 256;               // threads per CTA for every kernel
constexpr int kWarps = kBlock / 32;

// --------------------------------------------- programmatic dependent launch ---
//
// The streaming kernels are launched with programmatic stream serialization
// (launch_pdl): the next kernel on the stream may be scheduled onto SMs while
// this one drains, instead of after it has fully retired.  Every such kernel
// calls pdl_wait() before its first global-memory access: it returns once the
// preceding kernel on the stream has completed and its writes are visible,
// so the ordering the caller sees is exactly stream order.  pdl_trigger()
// (after the wait) lets the following kernel be scheduled as soon as every
// CTA of this grid has started.  After a non-kernel operation (memset, event,
// copy) or a kernel that never triggers, both are plain stream order.
#ifndef MOE_PDL
#define MOE_PDL 1
#endif

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = MOE_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ------------------------------------------------------------------ bf16 ---

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Two floats -> two bf16 (round to nearest even), `a` in the low half (the
// lower address), `b` in the high half.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
    f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
    f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
    uint4 v;
    v.x = pack_bf16x2(f[0], f[1]);
    v.y = pack_bf16x2(f[2], f[3]);
    v.z = pack_bf16x2(f[4], f[5]);
    v.w = pack_bf16x2(f[6], f[7]);
    return v;
}

// Router-dtype weight -> fp32 (exact widening for both dtypes).
__device__ __forceinline__ float load_weight(const void* w, int dtype, int64_t f) {
    if (dtype == MOE_DTYPE_F32) return static_cast<const float*>(w)[f];
    return __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(w)[f]) << 16);
}

// ------------------------------------------------------------ 16-B moves ---

// Read-only, single-use rows: non-coherent path, no L1 allocation.
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Row stores are never read back by the storing kernel: no L1 allocation
// (measured: Qwen3-shaped combine + backward 277.2 -> 275.2 us, dispatch
// 111.7 -> 111.0 us against plain stores; .cs streaming stores about the same).
__device__ __forceinline__ void st_vec(uint4* p, const uint4& v) {
    asm volatile("st.global.L1::no_allocate.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// 32-byte moves (sm_100 has 256-bit global loads and stores): two 16-byte
// vectors per instruction, for rows that are whole 32-byte vectors in
// 32-byte-aligned buffers.
struct alignas(32) Vec32 {
    uint4 lo, hi;
};

__device__ __forceinline__ Vec32 make_vec32_zero() {
    Vec32 v;
    v.lo = make_uint4(0u, 0u, 0u, 0u);
    v.hi = v.lo;
    return v;
}

__device__ __forceinline__ Vec32 ld_stream32(const uint4* p) {
    Vec32 v;
    asm volatile(
        "ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(v.lo.x), "=r"(v.lo.y), "=r"(v.lo.z), "=r"(v.lo.w), "=r"(v.hi.x), "=r"(v.hi.y),
          "=r"(v.hi.z), "=r"(v.hi.w)
        : "l"(p));
    return v;
}

__device__ __forceinline__ void st_vec32(uint4* p, const Vec32& v) {
    asm volatile("st.global.L1::no_allocate.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p),
                 "r"(v.lo.x), "r"(v.lo.y), "r"(v.lo.z), "r"(v.lo.w), "r"(v.hi.x), "r"(v.hi.y),
                 "r"(v.hi.z), "r"(v.hi.w)
                 : "memory");
}

// ------------------------------------------------------- bulk (TMA) copies ---
//
// Non-tensor bulk loads from global into shared memory done by the SM's
// copy engine, completing on an mbarrier (its transaction count).  Addresses
// and sizes are multiples of 16 bytes.  No multicast form is used anywhere.

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

// Makes mbarrier initialisation visible to the copy engine.
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// One arrival (no transaction bytes) of the calling thread.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// One bounded probe of phase `parity`; true once that phase has completed.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, unsigned bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_addr(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// ------------------------------------------------------------- warp/block ---

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

__device__ __forceinline__ void status_or(int32_t* status, int bits) {
    if (bits) atomicOr(status, bits);
}

// Warp-wide OR of `bits`, one atomic per warp (all 32 lanes must call).
__device__ __forceinline__ void warp_status_or(int32_t* status, int bits) {
    for (int d = 16; d > 0; d >>= 1) bits |= __shfl_xor_sync(kFull, bits, d);
    if ((threadIdx.x & 31) == 0) status_or(status, bits);
}

// In-place exclusive prefix sum of n <= kBlock*kPer ints in shared memory by
// the whole CTA (blockDim.x == kBlock); returns the total to every thread.
// `scratch` holds kWarps + 1 ints.  Ends with a __syncthreads().
template <int kPer>
__device__ int block_exclusive_scan(int* data, int n, int* scratch) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int begin = tid * kPer;
    int vals[kPer];
    int local = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        vals[i] = (begin + i < n) ? data[begin + i] : 0;
        local += vals[i];
    }
    int incl = local;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        int v = __shfl_up_sync(kFull, incl, d);
        if (lane >= d) incl += v;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int w = 0; w < kWarps; ++w) {
            int v = scratch[w];
            scratch[w] = run;
            run += v;
        }
        scratch[kWarps] = run;
    }
    __syncthreads();
    int run = scratch[warp] + incl - local;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        if (begin + i < n) data[begin + i] = run;
        run += vals[i];
    }
    const int total = scratch[kWarps];
    __syncthreads();
    return total;
}

// Largest e in [0, n) with a[e] <= v, for non-decreasing a (a[0] <= v).
__device__ __forceinline__ int upper_index(const int* a, int n, int v) {
    int lo = 0, hi = n;  // invariant: a[lo] <= v, answer in [lo, hi)
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (a[mid] <= v) lo = mid; else hi = mid;
    }
    return lo;
}

}  // namespace moe
