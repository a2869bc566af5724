// route_topk.cu -- router softmax + top-k, one warp per token.
//
// "Efficient and portable mixture-of-experts communication", "Introdução":
// the router yields a probability distribution over the experts; the top-K
// are chosen and weight the expert outputs.  Gating stays in its original
// precision (DeepSeek-V3 fragments): fp32 logits in, fp32 weights out.
//
// Each lane holds the logits e = i*32 + lane (a warp-wide load per i is one
// coalesced 128-byte line).  k rounds of warp arg-max under the order (logit
// descending, index ascending) pick the experts; a per-lane bit mask removes
// the winners.  The softmax denominator is summed in binary64 over all E
// experts and every weight is one binary64 quotient rounded once to fp32, so
// the result differs from any other correct binary64 evaluation by at most
// one fp32 ulp.
#include <cfloat>
#include <climits>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kRouteWarps = 8;  // tokens per CTA

struct Cand {
    float v;
    int e;  // INT_MAX: no candidate
};

__device__ __forceinline__ bool better(const Cand &a, const Cand &b)
{
    if (a.e == INT_MAX)
        return false;
    if (b.e == INT_MAX)
        return true;
    return a.v > b.v || (a.v == b.v && a.e < b.e);
}

template <int NPL>
__global__ void __launch_bounds__(kRouteWarps * 32)
    k_route_topk(const float *__restrict__ logits, int T, int E, int k, int renormalize,
                 int32_t *__restrict__ topk_idx, float *__restrict__ topk_w)
{
    const int lane = threadIdx.x & 31;
    const int g = blockIdx.x * kRouteWarps + (threadIdx.x >> 5);
    if (g >= T)
        return;  // warp-uniform
    const float *row = logits + static_cast<size_t>(g) * E;

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

    int my_e = 0;
    float my_v = 0.0f;
    float vmax = 0.0f;
    for (int j = 0; j < k; ++j) {
        Cand best{-FLT_MAX, INT_MAX};
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            // e grows with i: a strict '>' keeps the lower index on ties
            if (!((gone >> i) & 1u) && (best.e == INT_MAX || v[i] > best.v))
                best = Cand{v[i], i * 32 + lane};
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            Cand o;
            o.v = __shfl_xor_sync(kFullMask, best.v, off);
            o.e = __shfl_xor_sync(kFullMask, best.e, off);
            if (better(o, best))
                best = o;
        }
        // k <= E: every round has a winner
        if ((best.e & 31) == lane)
            gone |= 1u << (best.e >> 5);
        if (lane == j) {
            my_e = best.e;
            my_v = best.v;
        }
        if (j == 0)
            vmax = best.v;
    }

    const double m = static_cast<double>(vmax);
    double denom = 0.0;
#pragma unroll
    for (int i = 0; i < NPL; ++i)
        if (i * 32 + lane < E)
            denom += exp(static_cast<double>(v[i]) - m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        denom += __shfl_xor_sync(kFullMask, denom, off);

    const double num = (lane < k) ? exp(static_cast<double>(my_v) - m) : 0.0;
    if (renormalize) {
        double s = num;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            s += __shfl_xor_sync(kFullMask, s, off);
        denom = s;
    }
    if (lane < k) {
        topk_idx[static_cast<size_t>(g) * k + lane] = my_e;
        topk_w[static_cast<size_t>(g) * k + lane] = __double2float_rn(num / denom);
    }
}

template <int NPL>
cudaError_t launch(const float *logits, int T, int E, int k, int renormalize, int32_t *idx,
                   float *w, cudaStream_t s)
{
    const int grid = ceil_div(T, kRouteWarps);
    k_route_topk<NPL><<<grid, kRouteWarps * 32, 0, s>>>(logits, T, E, k, renormalize, idx, w);
    return cudaGetLastError();
}

}  // namespace

cudaError_t route_topk(const float *logits, int T, int E, int k, int renormalize,
                       int32_t *topk_idx, float *topk_w, cudaStream_t s)
{
    const int need = ceil_div(E, 32);
    if (need <= 1) return launch<1>(logits, T, E, k, renormalize, topk_idx, topk_w, s);
    if (need <= 2) return launch<2>(logits, T, E, k, renormalize, topk_idx, topk_w, s);
    if (need <= 4) return launch<4>(logits, T, E, k, renormalize, topk_idx, topk_w, s);
    if (need <= 8) return launch<8>(logits, T, E, k, renormalize, topk_idx, topk_w, s);
    if (need <= 12) return launch<12>(logits, T, E, k, renormalize, topk_idx, topk_w, s);
    if (need <= 16) return launch<16>(logits, T, E, k, renormalize, topk_idx, topk_w, s);
    if (need <= 24) return launch<24>(logits, T, E, k, renormalize, topk_idx, topk_w, s);
    return launch<32>(logits, T, E, k, renormalize, topk_idx, topk_w, s);
}

}  // namespace moe
