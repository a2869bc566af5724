// route_topk.cu -- router softmax + top-k, one warp per token (the per-token
// step is route_warp in route_dev.cuh).
//
// The extended form (shared experts, expert replicas; DeepSeek-V3 fragments:
// during decoding the shared expert is treated as a routed one that every
// token selects, and redundant experts replicate heavily loaded ones)
// appends the shared slots after the k routed ones and maps each logical
// expert through the caller's replica table in the same epilogue.
#include "common.cuh"
#include "kernels.cuh"
#include "route_dev.cuh"

namespace moe {

namespace {

constexpr int kRouteWarps = 8;  // tokens per CTA

// At most 1024 experts (NPL = 32) a lane holds 32 logits and their keys: the
// register budget is left open there (one CTA per SM suffices to fill the
// grid's few warps per token) so nothing spills.
template <int NPL, bool EX, int KT>
__global__ void __launch_bounds__(kRouteWarps * 32, NPL >= 24 ? 1 : 4)
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
    // release the next kernel at once: it still waits for this one to finish
    // before reading, so its CTAs only take idle SM slots early
    pdl_trigger();
    pdl_wait();

    int my_e;
    float my_w;
    route_warp<NPL, KT>(row, E, k, renormalize, my_e, my_w);
    if (!EX) {
        if (lane < k) {
            topk_idx[static_cast<size_t>(g) * k + lane] = my_e;
            topk_w[static_cast<size_t>(g) * k + lane] = my_w;
        }
    } else {
        // shared experts E .. E + n_shared - 1 follow the routed ones; every
        // logical expert maps to the replica chosen by the token's source rank
        const int kk = k + ex.n_shared;
        if (lane < kk) {
            const int l = (lane < k) ? my_e : E + (lane - k);
            const float wt = (lane < k) ? my_w : ex.shared_weight;
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
}

template <int NPL, int KT>
cudaError_t launch_kt(const float *logits, int T, int E, int k, int renormalize, int32_t *idx,
                      float *w, const RouteEx *ex, cudaStream_t s)
{
    const int grid = ceil_div(T, kRouteWarps);
    if (ex == nullptr)
        return launch_pdl(k_route_topk<NPL, false, KT>, dim3(grid), dim3(kRouteWarps * 32), 0, s,
                          logits, T, E, k, renormalize, idx, w, RouteEx{});
    return launch_pdl(k_route_topk<NPL, true, KT>, dim3(grid), dim3(kRouteWarps * 32), 0, s, logits,
                      T, E, k, renormalize, idx, w, *ex);
}

// k = 8 (the decode and prefill routers) unrolls its rounds: 7.4 -> 6.2 us
// for 4096 tokens at E = 256 (with the other changes of route_warp,
// 8.2 -> 6.2 us; prefill 32.8 -> 24.3 us, kimi 12.1 -> 8.4 us).
template <int NPL>
cudaError_t launch(const float *logits, int T, int E, int k, int renormalize, int32_t *idx,
                   float *w, const RouteEx *ex, cudaStream_t s)
{
    if (NPL >= 4 && k == 8)
        return launch_kt<NPL, (NPL >= 4 ? 8 : 0)>(logits, T, E, k, renormalize, idx, w, ex, s);
    return launch_kt<NPL, 0>(logits, T, E, k, renormalize, idx, w, ex, s);
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
