// route_dev.cuh -- the per-token router step (softmax + top-k) as a warp-wide
// device function, shared by the route kernel and the fused
// route -> layout -> dispatch kernel so both give the same bits.
//
// "Efficient and portable mixture-of-experts communication", "Introdução":
// the router yields a probability distribution over the experts; the top-K
// are chosen and weight the expert outputs.  Gating stays in its original
// precision (DeepSeek-V3 fragments): fp32 logits in, fp32 weights out.
//
// Each lane holds the logits e = i*32 + lane (a warp-wide load per i is one
// coalesced 128-byte line), as order-preserving 32-bit keys.  k rounds of
// warp arg-max under the order (logit descending, index ascending) pick the
// experts: one warp-wide max of the lanes' best keys and one warp-wide min of
// the indices holding it (redux.sync, a single instruction each), then the
// winner's key is cleared.
//
// The softmax is evaluated in fp32 with its error bounded (u = 2^-24):
//   d = l - m is split exactly into d_hi + d_lo (Knuth's TwoSum), so the
//   exponent sees no rounding of the difference; t = expf(d_hi) * (1 + d_lo)
//   has relative error <= 5u (expf is within 2 ulp = 4u, plus one rounding);
//   the denominator is a compensated (Neumaier) sum of the positive t, within
//   2u of their exact sum; w = t_j / S is one IEEE division (u).  Hence
//   |w - p| <= 13u * p (+ O(u^2)) for the exact probability p, i.e. within 16
//   fp32 ulps of the correctly rounded value; in practice 1-2 ulps.
#pragma once

#include <cfloat>

#include "common.cuh"

namespace moe {

// a + b == s + err exactly (Knuth's TwoSum; explicit _rn ops are never
// contracted or reassociated)
__device__ __forceinline__ void two_sum(float a, float b, float &s, float &err)
{
    s = __fadd_rn(a, b);
    const float bb = __fsub_rn(s, a);
    err = __fadd_rn(__fsub_rn(a, __fsub_rn(s, bb)), __fsub_rn(b, bb));
}

// Neumaier's compensated summation step: (sum + comp) absorbs t.
__device__ __forceinline__ void neumaier_add(float &sum, float &comp, float t)
{
    float s, err;
    two_sum(sum, t, s, err);
    sum = s;
    comp = __fadd_rn(comp, err);
}

// exp(l - m) for fp32 l <= m: the difference split exactly into hi + lo, the
// exponential of hi by expf, the first-order factor (1 + lo) applied with one
// fused multiply-add (|lo| <= 2^-24 |hi|, so the dropped lo^2/2 is far below
// the rounding of the result).
__device__ __forceinline__ float exp_diff(float l, float m)
{
    float hi, lo;
    two_sum(l, -m, hi, lo);
    if (hi < -104.0f)  // expf underflows to 0 (and keeps an overflowed hi from making NaN)
        return 0.0f;
    const float t = expf(hi);
    return __fmaf_rn(t, lo, t);
}

// Warp-wide compensated sum of (sum, comp) pairs.
__device__ __forceinline__ float warp_neumaier_total(float sum, float comp)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float os = __shfl_xor_sync(kFullMask, sum, off);
        const float oc = __shfl_xor_sync(kFullMask, comp, off);
        comp = __fadd_rn(comp, oc);
        neumaier_add(sum, comp, os);
    }
    return __fadd_rn(sum, comp);
}

// Route one token with the whole warp: on return lane j < k holds the j-th
// chosen expert (logit descending, index ascending among equal logits) in
// `my_e` and its weight in `my_w` (the softmax probability over all E, or
// over the k chosen ones with `renormalize`).  Other lanes' outputs are 0.
// NPL = logits per lane, NPL * 32 >= E.  Called by all 32 lanes.
template <int NPL>
__device__ __forceinline__ void route_warp(const float *__restrict__ row, int E, int k,
                                           int renormalize, int &my_e, float &my_w)
{
    const int lane = threadIdx.x & 31;
    float v[NPL];
    uint32_t gone = 0;  // bit i: element i past E
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = i * 32 + lane;
        if (e < E) {
            v[i] = __ldg(row + e);
        } else {
            v[i] = -FLT_MAX;
            gone |= 1u << i;
        }
    }

    // selection on order-preserving 32-bit keys: larger logit -> larger key,
    // -0 and +0 the same key (x + 0.0f turns -0 into +0); key 0 = taken/absent
    uint32_t key[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        if ((gone >> i) & 1u) {
            key[i] = 0u;
        } else {
            const uint32_t u = __float_as_uint(__fadd_rn(v[i], 0.0f));
            key[i] = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
        }
    }
    my_e = 0;
    float my_v = 0.0f;
    float vmax = 0.0f;
    for (int j = 0; j < k; ++j) {
        uint32_t best = 0u;
#pragma unroll
        for (int i = 0; i < NPL; ++i)
            best = max(best, key[i]);
        const uint32_t m = __reduce_max_sync(kFullMask, best);
        uint32_t cand = 0xffffffffu;
#pragma unroll
        for (int i = NPL - 1; i >= 0; --i)
            if (key[i] == m)
                cand = static_cast<uint32_t>(i * 32 + lane);
        const uint32_t e = __reduce_min_sync(kFullMask, cand);
        const int ei = static_cast<int>(e >> 5);
        float ve = 0.0f;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            if (i == ei && (e & 31u) == static_cast<uint32_t>(lane)) {
                key[i] = 0u;
            }
            if (i == ei)
                ve = v[i];
        }
        ve = __shfl_sync(kFullMask, ve, static_cast<int>(e & 31u));
        if (lane == j) {
            my_e = static_cast<int>(e);
            my_v = ve;
        }
        if (j == 0)
            vmax = ve;
    }

    // softmax over all E logits, in fp32 with compensated summation
    float sum = 0.0f, comp = 0.0f;
#pragma unroll
    for (int i = 0; i < NPL; ++i)
        if (i * 32 + lane < E)
            neumaier_add(sum, comp, exp_diff(v[i], vmax));
    float denom = warp_neumaier_total(sum, comp);

    const float num = (lane < k) ? exp_diff(my_v, vmax) : 0.0f;
    if (renormalize)
        denom = warp_neumaier_total(num, 0.0f);
    my_w = (lane < k) ? __fdiv_rn(num, denom) : 0.0f;
}

}  // namespace moe
