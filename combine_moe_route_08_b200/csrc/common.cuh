// common.cuh -- small device helpers shared by the kernels of libmoe_route.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_route.h"

namespace moe {

constexpr unsigned kFullMask = 0xffffffffu;

// First error wins: a kernel that finds a bad element records its code once.
__device__ __forceinline__ void report(int32_t *dev_status, int code)
{
    if (dev_status != nullptr)
        atomicCAS(dev_status, 0, code);
}

// 16-byte load that is not kept in L1 (each row is read exactly once).
__device__ __forceinline__ uint4 ld_stream_v4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 16-byte streaming store (evict-first: the receive buffers are far larger
// than L2 and are not read again by this library).
__device__ __forceinline__ void st_stream_v4(void *p, uint4 v)
{
    __stcs(reinterpret_cast<uint4 *>(p), v);
}

// The two bf16 values of a 32-bit word (low half = lower address) as floats;
// bf16 -> fp32 is exact (the bf16 bits are the top half of the fp32).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two fp32 values -> two OCP E4M3 codes, round to nearest even, saturating
// to +-448 (NaN -> 0x7F), by the hardware conversion.  `a` lands in the low
// byte (the lower address once stored little-endian).
__device__ __forceinline__ uint32_t e4m3x2(float a, float b)
{
    return static_cast<uint32_t>(
        __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

// Two fp32 values -> bf16x2 word, round to nearest even; `a` in the low half.
__device__ __forceinline__ uint32_t bf16x2_rn(float a, float b)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Programmatic dependent launch.  Every kernel of the library is launched
// with programmatic stream serialisation: it may start while the previous
// kernel on the stream drains.  pdl_wait() must come before the first read of
// anything an earlier kernel wrote; pdl_trigger() lets the next kernel launch
// once every CTA of this one has passed it (its own pdl_wait still waits for
// this kernel to finish and its memory to be visible).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ int round_up(int a, int b) { return ceil_div(a, b) * b; }

}  // namespace moe
