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
// coalesced 128-byte line), as order-preserving 32-bit keys, and tracks its
// own best and second-best key.  k rounds of warp arg-max under the order
// (logit descending, index ascending) pick the experts: one warp-wide max of
// the lanes' best keys and one warp-wide min of the expert ids holding it
// (redux.sync, a single instruction each); the winning lane promotes its
// second best, and rescans only when it has none left.
//
// The softmax is evaluated with its error bounded (u = 2^-24):
//   d = l - m is split exactly into d_hi + d_lo (Knuth's TwoSum), so the
//   exponent sees no rounding of the difference; t = expf(d_hi) * (1 + d_lo)
//   has relative error <= 5u (expf is within 2 ulp = 4u, plus one rounding);
//   the denominator sums the positive t in binary64 (at most 1024 terms of at
//   most 1: its error is below 2^-42 relative, far under u) and is rounded
//   once to binary32 (u); w = t_j / S is one IEEE division (u).  Hence
//   |w - p| <= 7u * p (+ O(u^2)) for the exact probability p; in practice
//   1-2 ulps.  Lane 0's total is broadcast, so all of a token's weights
//   share one denominator.
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

// Warp-wide binary64 sum, rounded once to binary32; lane 0's value for all.
__device__ __forceinline__ float warp_total_f64(double sum)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        sum = __dadd_rn(sum, __shfl_xor_sync(kFullMask, sum, off));
    return __shfl_sync(kFullMask, __double2float_rn(sum), 0);
}

// Order-preserving 32-bit key of a logit: larger logit -> larger key, -0 and
// +0 the same key (x + 0.0f turns -0 into +0); key 0 is never produced for a
// finite or infinite logit and marks a taken or absent slot.
__device__ __forceinline__ uint32_t logit_key(float x)
{
    const uint32_t u = __float_as_uint(__fadd_rn(x, 0.0f));
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The logit a key came from (the map is invertible; -0 comes back as +0,
// which gives the same softmax terms).
__device__ __forceinline__ float key_logit(uint32_t m)
{
    return __uint_as_float((m & 0x80000000u) ? (m & 0x7fffffffu) : ~m);
}

// Route one token with the whole warp: on return lane j < k holds the j-th
// chosen expert (logit descending, index ascending among equal logits) in
// `my_e` and its weight in `my_w` (the softmax probability over all E, or
// over the k chosen ones with `renormalize`).  Other lanes' outputs are 0.
// NPL = logits per lane, NPL * 32 >= E.  KT > 0: k == KT known at compile
// time (the rounds unroll); KT == 0: k at run time.  Called by all 32 lanes.
//
// Lane l holds experts l, l + 32, ...: hot experts of a skewed router (a
// Zipf-like bias on the lowest ids) fall on different lanes, so a lane
// rarely wins more rounds than its two best keys cover.  (Holding eight
// consecutive experts per lane, loaded as two 16-byte vectors, measured the
// same at dsv3 and prefill but 12.3 against 8.4 us at the skewed kimi
// workload: lane 0 won most rounds and rescanned.)
template <int NPL, int KT = 0>
__device__ __forceinline__ void route_warp(const float *__restrict__ row, int E, int k,
                                           int renormalize, int &my_e, float &my_w)
{
    const int lane = threadIdx.x & 31;
    float v[NPL];
    uint32_t key[NPL];
    uint32_t gone = 0;  // bit i: slot i taken or past E
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = i * 32 + lane;
        if (e < E) {
            v[i] = __ldg(row + e);
            key[i] = logit_key(v[i]);
        } else {
            v[i] = -FLT_MAX;
            key[i] = 0u;
            gone |= 1u << i;
        }
    }

    // Each lane keeps its best key b1 (slot i1) and, while known, its second
    // best b2 (order: key descending, slot ascending, so the lower expert
    // first among equal keys).  A round is one warp max of the lanes' bests
    // and one warp min of the expert ids holding it (redux.sync); the lane
    // whose expert won promotes its second best, and only a lane that wins
    // again with no second left rescans its remaining keys.
    uint32_t b1 = 0u, b2 = 0u;
    int i1 = 0, i2 = 0;
    auto top2 = [&]() {
        b1 = 0u;
        b2 = 0u;
        i1 = 0;
        i2 = 0;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const uint32_t kk = ((gone >> i) & 1u) ? 0u : key[i];
            if (kk > b1) {
                b2 = b1;
                i2 = i1;
                b1 = kk;
                i1 = i;
            } else if (kk > b2) {
                b2 = kk;
                i2 = i;
            }
        }
    };
    top2();
    my_e = 0;
    uint32_t my_key = 0u, m0 = 0u;
    const int nk = (KT > 0) ? KT : k;
#pragma unroll(KT > 0 ? KT : 1)
    for (int j = 0; j < nk; ++j) {
        const uint32_t m = __reduce_max_sync(kFullMask, b1);
        const uint32_t cand = (b1 == m) ? static_cast<uint32_t>(i1 * 32 + lane) : 0xffffffffu;
        const uint32_t e = __reduce_min_sync(kFullMask, cand);
        if (lane == j) {
            my_key = m;
            my_e = static_cast<int>(e);
        }
        if (j == 0)
            m0 = m;
        if (e == cand) {  // this lane's best was chosen: move to its next best
            gone |= 1u << i1;
            if (b2 != 0u) {
                b1 = b2;
                i1 = i2;
                b2 = 0u;  // unknown until needed
            } else {
                top2();  // taken keys are skipped
            }
        }
    }
    const float vmax = key_logit(m0);
    const float my_v = key_logit(my_key);

    // softmax over all E logits: fp32 terms, binary64 sum
    double sum = 0.0;
#pragma unroll
    for (int i = 0; i < NPL; ++i)
        if (i * 32 + lane < E)
            sum = __dadd_rn(sum, static_cast<double>(exp_diff(v[i], vmax)));
    float denom = warp_total_f64(sum);

    const float num = (lane < k) ? exp_diff(my_v, vmax) : 0.0f;
    if (renormalize)
        denom = warp_total_f64(static_cast<double>(num));
    my_w = (lane < k) ? __fdiv_rn(num, denom) : 0.0f;
}

}  // namespace moe
