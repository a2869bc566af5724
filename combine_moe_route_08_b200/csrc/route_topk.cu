// route_topk.cu -- router softmax + top-k, one warp per token.
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
// The extended form (shared experts, expert replicas; DeepSeek-V3 fragments:
// during decoding the shared expert is treated as a routed one that every
// token selects, and redundant experts replicate heavily loaded ones)
// appends the shared slots after the k routed ones and maps each logical
// expert through the caller's replica table in the same epilogue.
//
// The softmax is evaluated in fp32 with its error bounded (u = 2^-24):
//   d = l - m is split exactly into d_hi + d_lo (Knuth's TwoSum), so the
//   exponent sees no rounding of the difference; t = expf(d_hi) * (1 + d_lo)
//   has relative error <= 5u (expf is within 2 ulp = 4u, plus one rounding);
//   the denominator is a compensated (Neumaier) sum of the positive t, within
//   2u of their exact sum; w = t_j / S is one IEEE division (u).  Hence
//   |w - p| <= 13u * p (+ O(u^2)) for the exact probability p, i.e. within 16
//   fp32 ulps of the correctly rounded value; in practice 1-2 ulps.
#include <cfloat>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kRouteWarps = 8;  // tokens per CTA

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

template <int NPL, bool EX>
__global__ void __launch_bounds__(kRouteWarps * 32)
    k_route_topk(const float *__restrict__ logits, int T, int E, int k, int renormalize,
                 int32_t *__restrict__ topk_idx, float *__restrict__ topk_w, RouteEx ex)
{
    const int lane = threadIdx.x & 31;
    const int g = blockIdx.x * kRouteWarps + (threadIdx.x >> 5);
    if (g >= T) {
        pdl_wait();
        pdl_trigger();
        return;  // warp-uniform
    }
    const float *row = logits + static_cast<size_t>(g) * E;
    pdl_wait();

    float v[NPL];
    uint32_t gone = 0;  // bit i: element i taken or past E
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
    int my_e = 0;
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
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float os = __shfl_xor_sync(kFullMask, sum, off);
        const float oc = __shfl_xor_sync(kFullMask, comp, off);
        comp = __fadd_rn(comp, oc);
        neumaier_add(sum, comp, os);
    }
    float denom = __fadd_rn(sum, comp);

    const float num = (lane < k) ? exp_diff(my_v, vmax) : 0.0f;
    if (renormalize) {
        float ks = num, kc = 0.0f;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float os = __shfl_xor_sync(kFullMask, ks, off);
            const float oc = __shfl_xor_sync(kFullMask, kc, off);
            kc = __fadd_rn(kc, oc);
            neumaier_add(ks, kc, os);
        }
        denom = __fadd_rn(ks, kc);
    }
    if (!EX) {
        if (lane < k) {
            topk_idx[static_cast<size_t>(g) * k + lane] = my_e;
            topk_w[static_cast<size_t>(g) * k + lane] = __fdiv_rn(num, denom);
        }
    } else {
        // shared experts E .. E + n_shared - 1 follow the routed ones; every
        // logical expert maps to the replica chosen by the token's source rank
        const int kk = k + ex.n_shared;
        if (lane < kk) {
            const int l = (lane < k) ? my_e : E + (lane - k);
            const float wt = (lane < k) ? __fdiv_rn(num, denom) : ex.shared_weight;
            int phys = l;
            if (ex.replica_offsets != nullptr) {
                const int a = ex.replica_offsets[l], b = ex.replica_offsets[l + 1];
                if (a < 0 || b <= a || b > ex.n_replica_ids)
                    phys = -1;
                else
                    phys = ex.replica_ids[a + (g / ex.tokens_per_rank) % (b - a)];
            }
            if (phys < 0 || phys >= ex.E_phys) {
                report(ex.dev_status, MOE_ERR_INVALID_ARG);
                phys = -1;
            }
            topk_idx[static_cast<size_t>(g) * kk + lane] = phys;
            topk_w[static_cast<size_t>(g) * kk + lane] = wt;
        }
    }
    pdl_trigger();
}

template <int NPL>
cudaError_t launch(const float *logits, int T, int E, int k, int renormalize, int32_t *idx,
                   float *w, const RouteEx *ex, cudaStream_t s)
{
    const int grid = ceil_div(T, kRouteWarps);
    if (ex == nullptr)
        return launch_pdl(k_route_topk<NPL, false>, dim3(grid), dim3(kRouteWarps * 32), 0, s,
                          logits, T, E, k, renormalize, idx, w, RouteEx{});
    return launch_pdl(k_route_topk<NPL, true>, dim3(grid), dim3(kRouteWarps * 32), 0, s, logits,
                      T, E, k, renormalize, idx, w, *ex);
}

}  // namespace

cudaError_t route_topk(const float *logits, int T, int E, int k, int renormalize,
                       int32_t *topk_idx, float *topk_w, const RouteEx *ex, cudaStream_t s)
{
    const int need = ceil_div(E, 32);
    if (need <= 1) return launch<1>(logits, T, E, k, renormalize, topk_idx, topk_w, ex, s);
    if (need <= 2) return launch<2>(logits, T, E, k, renormalize, topk_idx, topk_w, ex, s);
    if (need <= 4) return launch<4>(logits, T, E, k, renormalize, topk_idx, topk_w, ex, s);
    if (need <= 8) return launch<8>(logits, T, E, k, renormalize, topk_idx, topk_w, ex, s);
    if (need <= 12) return launch<12>(logits, T, E, k, renormalize, topk_idx, topk_w, ex, s);
    if (need <= 16) return launch<16>(logits, T, E, k, renormalize, topk_idx, topk_w, ex, s);
    if (need <= 24) return launch<24>(logits, T, E, k, renormalize, topk_idx, topk_w, ex, s);
    return launch<32>(logits, T, E, k, renormalize, topk_idx, topk_w, ex, s);
}

}  // namespace moe
