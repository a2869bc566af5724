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

// The same quantisation for a thread holding 32 consecutive channels (four
// 16-byte words): the 4 threads of a 128-channel block are 4 consecutive
// lanes aligned to 4, so the block's amax is a 2-step xor shuffle.  The same
// amax, scale and divisions per channel as quant_e4m3_x16, so the same codes.
// Codes of channels 0-15 in q0, 16-31 in q1.  Called by all 32 lanes.
__device__ __forceinline__ void quant_e4m3_x32(const uint4 (&in)[4], uint4 &q0, uint4 &q1,
                                               float &s)
{
    float f[32];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const uint32_t wds[4] = {in[u].x, in[u].y, in[u].z, in[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[8 * u + 2 * i] = bf16_lo(wds[i]);
            f[8 * u + 2 * i + 1] = bf16_hi(wds[i]);
        }
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i)
        amax = fmaxf(amax, fabsf(f[i]));
    amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 2));
    s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
    uint32_t c[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t lo = e4m3x2(__fdiv_rn(f[4 * i], s), __fdiv_rn(f[4 * i + 1], s));
        const uint32_t hi = e4m3x2(__fdiv_rn(f[4 * i + 2], s), __fdiv_rn(f[4 * i + 3], s));
        c[i] = lo | (hi << 16);
    }
    q0 = make_uint4(c[0], c[1], c[2], c[3]);
    q1 = make_uint4(c[4], c[5], c[6], c[7]);
}

constexpr int kPrefetchPiece = 32768;  // bytes per L2 prefetch (a multiple of 16)

// Share `share` of `shares` of the bulk L2 prefetches covering
// [p, p + bytes): the pieces of kPrefetchPiece bytes whose index is congruent
// to `share`, issued by the CTA's threads in turn.  p 16-byte aligned, bytes
// a multiple of 16 and below 2^46.  TMA's untiled prefetch is fire-and-forget: no register,
// no shared memory, nothing to wait for.  It only warms L2, the point of
// coherence, so it can never expose stale data; lines evicted again are read
// from HBM as usual.
__device__ __forceinline__ void l2_prefetch_share(const void *p, int64_t bytes, int share,
                                                  int shares)
{
    // at most L2-sized ranges: piece indices fit in 32 bits
    const int n = static_cast<int>((bytes + kPrefetchPiece - 1) / kPrefetchPiece);
    const uint8_t *base = static_cast<const uint8_t *>(p);
    for (int i = static_cast<int>(threadIdx.x) * shares + share; i < n;
         i += static_cast<int>(blockDim.x) * shares) {
        const int64_t off = static_cast<int64_t>(i) * kPrefetchPiece;
        const uint32_t size =
            (i == n - 1) ? static_cast<uint32_t>(bytes - off) : static_cast<uint32_t>(kPrefetchPiece);
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(base + off), "r"(size)
                     : "memory");
    }
}

}  // namespace moe
