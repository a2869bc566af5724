// dispatch_dev.cuh -- the block-scaled FP8 quantisation of 16 channels, shared
// by the dispatch kernel and the fused route -> layout -> dispatch kernel.
//
// DeepSeek-V3 fragments: activations are scaled per token per 128 channels
// (1x128 tiles); "Enabling trillion-parameter models on AWS EFA",
// "Dağıtım/Birleştirme Gecikmesi": block-scaled fp8 dispatch.
#pragma once

#include "common.cuh"

namespace moe {

// A thread holds 16 consecutive bf16 channels (two 16-byte words); the 8
// threads of one 128-channel block are 8 consecutive lanes aligned to 8, so
// the block's amax is a 3-step xor shuffle.  s = amax / 448 (1 for an
// all-zero block) and every x / s are IEEE binary32 divisions (__fdiv_rn),
// then the hardware converts to e4m3 with RNE + saturation.  Returns the 16
// codes (channel order = byte order) and the block scale in `s`.  Called by
// all 32 lanes (an inactive lane passes zeros).
__device__ __forceinline__ uint4 quant_e4m3_x16(uint4 a, uint4 b, float &s)
{
    const uint32_t wds[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    float f[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        f[2 * i] = bf16_lo(wds[i]);
        f[2 * i + 1] = bf16_hi(wds[i]);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i)
        amax = fmaxf(amax, fabsf(f[i]));
    amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 4));
    s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);

    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t lo = e4m3x2(__fdiv_rn(f[4 * i], s), __fdiv_rn(f[4 * i + 1], s));
        const uint32_t hi = e4m3x2(__fdiv_rn(f[4 * i + 2], s), __fdiv_rn(f[4 * i + 3], s));
        c[i] = lo | (hi << 16);
    }
    return make_uint4(c[0], c[1], c[2], c[3]);
}

}  // namespace moe
