// common.cuh -- shared helpers of the lowbit CUDA library (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "lowbit.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "liblowbit is built for sm_100a (B200) only"
#endif

namespace lowbit {

constexpr int kWarp = 32;

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

inline lowbit_status launch_status()
{
    return cudaGetLastError() == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b)
{
    return __uint_as_float(b << 16);  // bf16 is the top half of an fp32
}

__device__ __forceinline__ float f16_bits_to_float(uint16_t h)
{
    return __half2float(__ushort_as_half(h));
}

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Integer sum over the warp in one reduction instruction (wraps mod 2^32
// like a chain of adds).
__device__ __forceinline__ int warp_sum_int(int v) { return __reduce_add_sync(0xffffffffu, v); }

// Maximum of non-negative finite floats over the warp in one reduction:
// their bit patterns order like unsigned integers.
__device__ __forceinline__ float warp_max_nonneg(float v)
{
    return __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(v)));
}

// Programmatic dependent launch: let the next kernel on the stream start its
// independent prologue early, and wait for the previous kernel's results.
__device__ __forceinline__ void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_primary()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Launch with the programmatic-stream-serialisation attribute so that a
// kernel which calls pdl_wait_primary() before touching dependent memory may
// overlap its prologue with the tail of the previous kernel.  LOWBIT_PDL=0
// at build time launches without it (plain stream order; for measurement).
#ifndef LOWBIT_PDL
#define LOWBIT_PDL 1
#endif
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = LOWBIT_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace lowbit
