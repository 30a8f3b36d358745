// Shared device/host helpers of the B200 ZO library (no method arithmetic here).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "kernels.h"

namespace zo {

__device__ __forceinline__ float ld_elem(const void* p, size_t i, int t) {
    return t == E_F32 ? static_cast<const float*>(p)[i]
                      : __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
}

__device__ __forceinline__ void st_elem(void* p, size_t i, int t, float v) {
    if (t == E_F32) static_cast<float*>(p)[i] = v;
    else static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Block-wide sum for blockDim.x a multiple of 32 (<= 1024); every thread gets the result.
__device__ __forceinline__ float block_sum(float v, float* red /* >= 32 floats */) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) red[w] = v;
    __syncthreads();
    float s = lane < nw ? red[lane] : 0.f;
    return warp_sum(s);
}

// Block-wide max, same contract as block_sum.
__device__ __forceinline__ float block_max(float v, float* red /* >= 32 floats */) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_max(v);
    __syncthreads();
    if (lane == 0) red[w] = v;
    __syncthreads();
    float s = lane < nw ? red[lane] : -3.0e38f;
    return warp_max(s);
}

inline unsigned cdiv(long long a, long long b) { return (unsigned)((a + b - 1) / b); }

// ---- debug build (ZO_DEBUG): device bounds checks -------------------------------------
// ZO_DCHECK(cond, bit) is `cond` in the debug build, where a failed check also ORs `bit` into
// the translation unit's debug word and the caller skips the access; in the release build it
// is `true` and compiles away.  No check traps.  A translation unit that checks places
// ZO_DEBUG_WORD(reader) at namespace scope before its kernels: the word, and a host function
// `unsigned reader(bool clear)` that returns it (0 in the release build).
#ifdef ZO_DEBUG
#define ZO_DCHECK(cond, bit) ((cond) ? true : (atomicOr(&g_zo_debug_word, (unsigned)(bit)), false))
#define ZO_DEBUG_WORD(reader)                                                               \
    static __device__ unsigned int g_zo_debug_word = 0;                                     \
    unsigned reader(bool clear) {                                                           \
        unsigned v = 0;                                                                     \
        if (cudaMemcpyFromSymbol(&v, g_zo_debug_word, sizeof(v)) != cudaSuccess) return ~0u; \
        if (clear) {                                                                        \
            const unsigned z = 0;                                                           \
            cudaMemcpyToSymbol(g_zo_debug_word, &z, sizeof(z));                             \
        }                                                                                   \
        return v;                                                                           \
    }
#else
#define ZO_DCHECK(cond, bit) true
#define ZO_DEBUG_WORD(reader) \
    unsigned reader(bool) { return 0; }
#endif

// Programmatic dependent launch: a kernel launched with launch_pdl may be scheduled while the
// kernel before it on the stream still runs; grid_dep_wait() blocks until that kernel has
// finished and its writes are visible (a no-op for an ordinary launch), grid_dep_launch()
// lets the next such kernel be scheduled early.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace zo
