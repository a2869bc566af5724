// abi.cu -- the extern "C" entry points of libmoe_route.so (declared, with
// their sources and contracts, in include/moe_route.h).  Every argument is
// checked here, on the host, before anything is enqueued; the kernels then
// only see in-range sizes and aligned pointers.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.cuh"
#include "moe_route.h"

namespace {

constexpr int kMaxE = 1024;
constexpr int kMaxK = 32;
constexpr int64_t kMaxIndex = INT32_MAX;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool valid_tk(int T, int k) { return T >= 0 && k >= 1 && k <= kMaxK && static_cast<int64_t>(T) * k < kMaxIndex; }

int launched(cudaError_t err) { return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

cudaStream_t as_stream(void *s) { return static_cast<cudaStream_t>(s); }

// Dispatch/combine: shared checks of the per-slot arguments.
int check_rows_args(int T, int H, int k, const void *dispatch_pos, int64_t rows)
{
    if (!valid_tk(T, k) || H < 8 || H % 8 != 0 || rows < 0 || rows >= kMaxIndex)
        return MOE_ERR_INVALID_ARG;
    if (T > 0 && (dispatch_pos == nullptr || !aligned(dispatch_pos, 4)))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

bool valid_layout_sizes(int T, int k, int E, int R)
{
    return valid_tk(T, k) && E >= 1 && E <= kMaxE && k <= E && R >= 1 && R <= E && E % R == 0 &&
           T % R == 0;
}

// The argument checks of each entry point, apart from its launch, so that the
// host-buffer entry points can check every step before enqueuing anything.
// They return a status, or kNothing: valid, and no kernel to launch (T == 0).
constexpr int kNothing = -1;

int done(int st) { return st == kNothing ? MOE_OK : st; }

int route_topk_args(const float *logits, int T, int E, int k, const int32_t *topk_idx,
                    const float *topk_w)
{
    if (!valid_tk(T, k) || E < 1 || E > kMaxE || k > E)
        return MOE_ERR_INVALID_ARG;
    if (T == 0)
        return kNothing;
    if (!logits || !topk_idx || !topk_w || !aligned(logits, 4) || !aligned(topk_idx, 4) ||
        !aligned(topk_w, 4))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// (the layout always launches: with T == 0 it still writes zero counts)
int layout_args(const int32_t *topk_idx, int T, int k, int E, int R, int capacity, int64_t rows,
                const int32_t *expert_counts, const int32_t *expert_src_counts,
                const int32_t *rank_counts, const int32_t *expert_offsets,
                const int32_t *dispatch_pos, const int32_t *recv_src, const void *workspace,
                size_t ws_bytes, const int32_t *dev_status)
{
    if (!valid_layout_sizes(T, k, E, R) || capacity < 0 || rows < 0 || rows >= kMaxIndex)
        return MOE_ERR_INVALID_ARG;
    const int64_t needed = (capacity == 0) ? static_cast<int64_t>(T) * k
                                           : static_cast<int64_t>(E) * capacity;
    if (rows < needed)
        return MOE_ERR_INVALID_ARG;
    const void *arrays[] = {expert_counts, expert_src_counts, rank_counts, expert_offsets};
    for (const void *p : arrays)
        if (!p || !aligned(p, 4))
            return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!topk_idx || !dispatch_pos || !aligned(topk_idx, 4) || !aligned(dispatch_pos, 4)))
        return MOE_ERR_INVALID_ARG;
    if (rows > 0 && (!recv_src || !aligned(recv_src, 4)))
        return MOE_ERR_INVALID_ARG;
    if (dev_status && !aligned(dev_status, 4))
        return MOE_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256) ||
        ws_bytes < moe::layout_workspace_bytes(moe::layout_geom(T, k, E, R)))
        return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

int dispatch_bf16_args(const uint16_t *x, int T, int H, int k, const int32_t *dispatch_pos,
                       const uint16_t *recv_x, int64_t rows, const int32_t *dev_status)
{
    const int st = check_rows_args(T, H, k, dispatch_pos, rows);
    if (st != MOE_OK)
        return st;
    if (T == 0)
        return kNothing;
    if (!x || !recv_x || !aligned(x, 16) || !aligned(recv_x, 16) ||
        (dev_status && !aligned(dev_status, 4)))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

int dispatch_fp8_args(const uint16_t *x, int T, int H, int k, const int32_t *dispatch_pos,
                      const uint8_t *recv_q, const float *recv_scale, int64_t rows,
                      const int32_t *dev_status)
{
    const int st = check_rows_args(T, H, k, dispatch_pos, rows);
    if (st != MOE_OK)
        return st;
    if (H % 128 != 0)
        return MOE_ERR_UNSUPPORTED;
    if (T == 0)
        return kNothing;
    if (!x || !recv_q || !recv_scale || !aligned(x, 16) || !aligned(recv_q, 16) ||
        !aligned(recv_scale, 4) || (dev_status && !aligned(dev_status, 4)))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

int combine_bf16_args(const uint16_t *y, const int32_t *dispatch_pos, const float *topk_w, int T,
                      int H, int k, int64_t rows, const uint16_t *out, const int32_t *dev_status)
{
    const int st = check_rows_args(T, H, k, dispatch_pos, rows);
    if (st != MOE_OK)
        return st;
    if (T == 0)
        return kNothing;
    if (!out || !topk_w || !aligned(out, 16) || !aligned(topk_w, 4) ||
        (dev_status && !aligned(dev_status, 4)))
        return MOE_ERR_INVALID_ARG;
    if (rows > 0 && (!y || !aligned(y, 16)))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

int combine_fp8_args(const uint8_t *y_q, const float *y_scale, const int32_t *dispatch_pos,
                     const float *topk_w, int T, int H, int k, int64_t rows, const uint16_t *out,
                     const int32_t *dev_status)
{
    const int st = check_rows_args(T, H, k, dispatch_pos, rows);
    if (st != MOE_OK)
        return st;
    if (H % 128 != 0)
        return MOE_ERR_UNSUPPORTED;
    if (T == 0)
        return kNothing;
    if (!out || !topk_w || !aligned(out, 16) || !aligned(topk_w, 4) ||
        (dev_status && !aligned(dev_status, 4)))
        return MOE_ERR_INVALID_ARG;
    if (rows > 0 && (!y_q || !y_scale || !aligned(y_q, 16) || !aligned(y_scale, 4)))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

}  // namespace

extern "C" {

const char *moe_status_string(int status)
{
    switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_CAPACITY: return "MOE_ERR_CAPACITY";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    default: return "MOE_ERR_UNKNOWN";
    }
}

int moe_route_topk(const float *logits, int T, int E, int k, int renormalize, int32_t *topk_idx,
                   float *topk_w, void *stream)
{
    const int st = route_topk_args(logits, T, E, k, topk_idx, topk_w);
    if (st != MOE_OK)
        return done(st);
    return launched(moe::route_topk(logits, T, E, k, renormalize != 0, topk_idx, topk_w, nullptr,
                                    as_stream(stream)));
}

int moe_route_topk_ex(const float *logits, int T, int E, int k, int renormalize, int n_shared,
                      float shared_weight, const int32_t *replica_offsets,
                      const int32_t *replica_ids, int n_replica_ids, int E_phys,
                      int tokens_per_rank, int32_t *topk_idx, float *topk_w, int32_t *dev_status,
                      void *stream)
{
    if (n_shared < 0 || n_shared > kMaxK || !valid_tk(T, k + n_shared) || k < 1 || E < 1 ||
        E > kMaxE || k > E || E_phys < 1 || tokens_per_rank < 1)
        return MOE_ERR_INVALID_ARG;
    if (replica_offsets != nullptr &&
        (replica_ids == nullptr || n_replica_ids < 1 || !aligned(replica_offsets, 4) ||
         !aligned(replica_ids, 4)))
        return MOE_ERR_INVALID_ARG;
    if (replica_offsets == nullptr && E_phys < E + n_shared)
        return MOE_ERR_INVALID_ARG;
    if (T == 0)
        return MOE_OK;
    if (!logits || !topk_idx || !topk_w || !aligned(logits, 4) || !aligned(topk_idx, 4) ||
        !aligned(topk_w, 4) || (dev_status && !aligned(dev_status, 4)))
        return MOE_ERR_INVALID_ARG;
    const moe::RouteEx ex{n_shared, shared_weight, replica_offsets, replica_ids, n_replica_ids,
                          E_phys, tokens_per_rank, dev_status};
    return launched(moe::route_topk(logits, T, E, k, renormalize != 0, topk_idx, topk_w, &ex,
                                    as_stream(stream)));
}

size_t moe_layout_workspace_bytes(int T, int k, int E, int R)
{
    if (!valid_layout_sizes(T, k, E, R))
        return 0;
    return moe::layout_workspace_bytes(moe::layout_geom(T, k, E, R));
}

int moe_dispatch_layout_launches(int T, int k, int E, int R)
{
    if (!valid_layout_sizes(T, k, E, R))
        return 0;
    return moe::layout_launches(moe::layout_geom(T, k, E, R));
}

int moe_dispatch_layout(const int32_t *topk_idx, int T, int k, int E, int R, int capacity,
                        int64_t rows, int32_t *expert_counts, int32_t *expert_src_counts,
                        int32_t *rank_counts, int32_t *expert_offsets, int32_t *dispatch_pos,
                        int32_t *recv_src, void *workspace, size_t ws_bytes, int32_t *dev_status,
                        void *stream)
{
    const int st = layout_args(topk_idx, T, k, E, R, capacity, rows, expert_counts,
                               expert_src_counts, rank_counts, expert_offsets, dispatch_pos,
                               recv_src, workspace, ws_bytes, dev_status);
    if (st != MOE_OK)
        return st;
    return launched(moe::dispatch_layout(topk_idx, moe::layout_geom(T, k, E, R), capacity, rows,
                                         expert_counts, expert_src_counts, rank_counts,
                                         expert_offsets, dispatch_pos, recv_src, nullptr,
                                         workspace, dev_status, as_stream(stream)));
}

int moe_dispatch_layout_private(const int32_t *topk_idx, int T, int k, int E, int R, int max_m,
                                int64_t rows, int32_t *expert_counts, int32_t *expert_src_counts,
                                int32_t *rank_counts, int32_t *expert_offsets,
                                int32_t *dispatch_pos, int32_t *recv_src, int32_t *private_pos,
                                void *workspace, size_t ws_bytes, int32_t *dev_status,
                                void *stream)
{
    if (!valid_layout_sizes(T, k, E, R) || max_m < 1 || rows < static_cast<int64_t>(T) * k ||
        rows >= kMaxIndex || static_cast<int64_t>(E) * R * max_m >= kMaxIndex)
        return MOE_ERR_INVALID_ARG;
    const void *arrays[] = {expert_counts, expert_src_counts, rank_counts, expert_offsets};
    for (const void *p : arrays)
        if (!p || !aligned(p, 4))
            return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!topk_idx || !dispatch_pos || !private_pos || !aligned(topk_idx, 4) ||
                  !aligned(dispatch_pos, 4) || !aligned(private_pos, 4)))
        return MOE_ERR_INVALID_ARG;
    if (rows > 0 && (!recv_src || !aligned(recv_src, 4)))
        return MOE_ERR_INVALID_ARG;
    if (dev_status && !aligned(dev_status, 4))
        return MOE_ERR_INVALID_ARG;
    moe::LayoutGeom g = moe::layout_geom(T, k, E, R);
    g.max_m = max_m;
    if (!workspace || !aligned(workspace, 256) || ws_bytes < moe::layout_workspace_bytes(g))
        return MOE_ERR_WORKSPACE;
    return launched(moe::dispatch_layout(topk_idx, g, 0, rows, expert_counts, expert_src_counts,
                                         rank_counts, expert_offsets, dispatch_pos, recv_src,
                                         private_pos, workspace, dev_status, as_stream(stream)));
}

int moe_compact_fp8(const uint8_t *priv_q, const float *priv_scale, int64_t private_rows,
                    const int32_t *private_pos, const int32_t *dispatch_pos, int T, int H, int k,
                    uint8_t *recv_q, float *recv_scale, int64_t rows, int32_t *dev_status,
                    void *stream)
{
    const int st = check_rows_args(T, H, k, dispatch_pos, rows);
    if (st != MOE_OK)
        return st;
    if (H % 128 != 0)
        return MOE_ERR_UNSUPPORTED;
    if (private_rows < 0 || private_rows >= kMaxIndex)
        return MOE_ERR_INVALID_ARG;
    if (T == 0)
        return MOE_OK;
    if (!priv_q || !priv_scale || !private_pos || !recv_q || !recv_scale || !aligned(priv_q, 16) ||
        !aligned(recv_q, 16) || !aligned(priv_scale, 4) || !aligned(recv_scale, 4) ||
        !aligned(private_pos, 4) || (dev_status && !aligned(dev_status, 4)))
        return MOE_ERR_INVALID_ARG;
    return launched(moe::compact_fp8(priv_q, priv_scale, private_rows, private_pos, dispatch_pos, T,
                                     H, k, recv_q, recv_scale, rows, dev_status,
                                     as_stream(stream)));
}

int moe_compact_bf16(const uint16_t *priv_x, int64_t private_rows, const int32_t *private_pos,
                     const int32_t *dispatch_pos, int T, int H, int k, uint16_t *recv_x,
                     int64_t rows, int32_t *dev_status, void *stream)
{
    const int st = check_rows_args(T, H, k, dispatch_pos, rows);
    if (st != MOE_OK)
        return st;
    if (private_rows < 0 || private_rows >= kMaxIndex)
        return MOE_ERR_INVALID_ARG;
    if (T == 0)
        return MOE_OK;
    if (!priv_x || !private_pos || !recv_x || !aligned(priv_x, 16) || !aligned(recv_x, 16) ||
        !aligned(private_pos, 4) || (dev_status && !aligned(dev_status, 4)))
        return MOE_ERR_INVALID_ARG;
    return launched(moe::compact_bf16(priv_x, private_rows, private_pos, dispatch_pos, T, H, k,
                                      recv_x, rows, dev_status, as_stream(stream)));
}

int moe_dispatch_bf16(const uint16_t *x, int T, int H, int k, const int32_t *dispatch_pos,
                      uint16_t *recv_x, int64_t rows, int32_t *dev_status, void *stream)
{
    const int st = dispatch_bf16_args(x, T, H, k, dispatch_pos, recv_x, rows, dev_status);
    if (st != MOE_OK)
        return done(st);
    return launched(moe::dispatch_bf16(x, T, H, k, dispatch_pos, recv_x, rows, dev_status,
                                       as_stream(stream)));
}

int moe_dispatch_fp8(const uint16_t *x, int T, int H, int k, const int32_t *dispatch_pos,
                     uint8_t *recv_q, float *recv_scale, int64_t rows, int32_t *dev_status,
                     void *stream)
{
    const int st = dispatch_fp8_args(x, T, H, k, dispatch_pos, recv_q, recv_scale, rows,
                                     dev_status);
    if (st != MOE_OK)
        return done(st);
    return launched(moe::dispatch_fp8(x, T, H, k, dispatch_pos, recv_q, recv_scale, rows, 0,
                                      dev_status, as_stream(stream)));
}

int moe_dispatch_fp8_ex(const uint16_t *x, int T, int H, int k, const int32_t *dispatch_pos,
                        uint8_t *recv_q, float *recv_scale, int64_t rows, int scale_layout,
                        int64_t scale_ld, int32_t *dev_status, void *stream)
{
    if (scale_layout == MOE_SCALE_ROW_MAJOR)
        return moe_dispatch_fp8(x, T, H, k, dispatch_pos, recv_q, recv_scale, rows, dev_status,
                                stream);
    if (scale_layout != MOE_SCALE_COL_MAJOR || scale_ld < rows || scale_ld % 4 != 0 ||
        scale_ld >= kMaxIndex)
        return MOE_ERR_INVALID_ARG;
    const int st = check_rows_args(T, H, k, dispatch_pos, rows);
    if (st != MOE_OK)
        return st;
    if (H % 128 != 0)
        return MOE_ERR_UNSUPPORTED;
    if (T == 0)
        return MOE_OK;
    if (!x || !recv_q || !recv_scale || !aligned(x, 16) || !aligned(recv_q, 16) ||
        !aligned(recv_scale, 16) || (dev_status && !aligned(dev_status, 4)))
        return MOE_ERR_INVALID_ARG;
    return launched(moe::dispatch_fp8(x, T, H, k, dispatch_pos, recv_q, recv_scale, rows, scale_ld,
                                      dev_status, as_stream(stream)));
}

int moe_combine_bf16(const uint16_t *y, const int32_t *dispatch_pos, const float *topk_w, int T,
                     int H, int k, int64_t rows, uint16_t *out, int32_t *dev_status, void *stream)
{
    const int st = combine_bf16_args(y, dispatch_pos, topk_w, T, H, k, rows, out, dev_status);
    if (st != MOE_OK)
        return done(st);
    return launched(moe::combine_bf16(y, dispatch_pos, topk_w, T, H, k, rows, out, dev_status,
                                      as_stream(stream)));
}

int moe_combine_bf16_long_form(int T, int H, int k)
{
    if (!valid_tk(T, k) || H < 8 || H % 8 != 0)
        return 0;
    return moe::combine_bf16_long_form(T, H, k) ? 1 : 0;
}

size_t moe_route_dispatch_workspace_bytes(int T, int k, int E, int R)
{
    if (!valid_layout_sizes(T, k, E, R))
        return 0;
    return moe::route_dispatch_workspace_bytes(T, k, E, R);
}

// The fused launch's argument checks (the workspace size is checked by the
// launch itself, against the geometry of the current device).
static int route_dispatch_args(const float *logits, int T, int E, int k, int R, int capacity,
                               const uint16_t *x, int H, bool fp8, const int32_t *topk_idx,
                               const float *topk_w, const int32_t *expert_counts,
                               const int32_t *expert_src_counts, const int32_t *rank_counts,
                               const int32_t *expert_offsets, const int32_t *dispatch_pos,
                               const int32_t *recv_src, const void *recv,
                               const float *recv_scale, int64_t rows, const void *workspace,
                               const int32_t *dev_status, const moe::RouteEx *ex)
{
    // the layout's view: slots per token and experts after the extension
    const int kl = k + (ex ? ex->n_shared : 0);
    const int El = ex ? ex->E_phys : E;
    if (ex && (E < 1 || E > kMaxE || k < 1 || k > E))
        return MOE_ERR_INVALID_ARG;
    if (!valid_layout_sizes(T, kl, El, R) || capacity < 0 || rows < 0 || rows >= kMaxIndex ||
        H < 8 || H % 8 != 0 || H > (1 << 20) || static_cast<int64_t>(T) * H > (int64_t(1) << 40))
        return MOE_ERR_INVALID_ARG;
    if ((fp8 && H % 128 != 0) || (!fp8 && H < 64))
        return MOE_ERR_UNSUPPORTED;
    const int64_t needed = (capacity == 0) ? static_cast<int64_t>(T) * kl
                                           : static_cast<int64_t>(El) * capacity;
    if (rows < needed)
        return MOE_ERR_INVALID_ARG;
    const void *arrays[] = {expert_counts, expert_src_counts, rank_counts, expert_offsets};
    for (const void *p : arrays)
        if (!p || !aligned(p, 4))
            return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!logits || !x || !topk_idx || !topk_w || !dispatch_pos || !aligned(logits, 4) ||
                  !aligned(x, 16) || !aligned(topk_idx, 4) || !aligned(topk_w, 4) ||
                  !aligned(dispatch_pos, 4)))
        return MOE_ERR_INVALID_ARG;
    if (rows > 0 && (!recv_src || !recv || !aligned(recv_src, 4) || !aligned(recv, 16) ||
                     (fp8 && (!recv_scale || !aligned(recv_scale, 4)))))
        return MOE_ERR_INVALID_ARG;
    if (dev_status && !aligned(dev_status, 4))
        return MOE_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256))
        return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

static int route_dispatch_common(const float *logits, int T, int E, int k, int renormalize, int R,
                                 int capacity, const uint16_t *x, int H, bool fp8,
                                 int32_t *topk_idx, float *topk_w, int32_t *expert_counts,
                                 int32_t *expert_src_counts, int32_t *rank_counts,
                                 int32_t *expert_offsets, int32_t *dispatch_pos,
                                 int32_t *recv_src, void *recv, float *recv_scale, int64_t rows,
                                 void *workspace, size_t ws_bytes, int32_t *dev_status,
                                 void *stream, const moe::RouteEx *ex = nullptr)
{
    const int st = route_dispatch_args(logits, T, E, k, R, capacity, x, H, fp8, topk_idx, topk_w,
                                       expert_counts, expert_src_counts, rank_counts,
                                       expert_offsets, dispatch_pos, recv_src, recv, recv_scale,
                                       rows, workspace, dev_status, ex);
    if (st != MOE_OK)
        return st;
    bool small = false;
    const cudaError_t err = moe::route_dispatch(
        logits, T, E, k, renormalize != 0, R, capacity, x, H, fp8, topk_idx, topk_w, expert_counts,
        expert_src_counts, rank_counts, expert_offsets, dispatch_pos, recv_src, recv, recv_scale,
        rows, workspace, ws_bytes, dev_status, as_stream(stream), &small, ex);
    if (small)
        return MOE_ERR_WORKSPACE;
    return launched(err);
}

int moe_route_dispatch_fp8(const float *logits, int T, int E, int k, int renormalize, int R,
                           int capacity, const uint16_t *x, int H, int32_t *topk_idx,
                           float *topk_w, int32_t *expert_counts, int32_t *expert_src_counts,
                           int32_t *rank_counts, int32_t *expert_offsets, int32_t *dispatch_pos,
                           int32_t *recv_src, uint8_t *recv_q, float *recv_scale, int64_t rows,
                           void *workspace, size_t ws_bytes, int32_t *dev_status, void *stream)
{
    return route_dispatch_common(logits, T, E, k, renormalize, R, capacity, x, H, true, topk_idx,
                                 topk_w, expert_counts, expert_src_counts, rank_counts,
                                 expert_offsets, dispatch_pos, recv_src, recv_q, recv_scale, rows,
                                 workspace, ws_bytes, dev_status, stream);
}

int moe_route_dispatch_bf16(const float *logits, int T, int E, int k, int renormalize, int R,
                            int capacity, const uint16_t *x, int H, int32_t *topk_idx,
                            float *topk_w, int32_t *expert_counts, int32_t *expert_src_counts,
                            int32_t *rank_counts, int32_t *expert_offsets, int32_t *dispatch_pos,
                            int32_t *recv_src, uint16_t *recv_x, int64_t rows, void *workspace,
                            size_t ws_bytes, int32_t *dev_status, void *stream)
{
    return route_dispatch_common(logits, T, E, k, renormalize, R, capacity, x, H, false, topk_idx,
                                 topk_w, expert_counts, expert_src_counts, rank_counts,
                                 expert_offsets, dispatch_pos, recv_src, recv_x, nullptr, rows,
                                 workspace, ws_bytes, dev_status, stream);
}

int moe_combine_fp8(const uint8_t *y_q, const float *y_scale, const int32_t *dispatch_pos,
                    const float *topk_w, int T, int H, int k, int64_t rows, uint16_t *out,
                    int32_t *dev_status, void *stream)
{
    const int st = combine_fp8_args(y_q, y_scale, dispatch_pos, topk_w, T, H, k, rows, out,
                                     dev_status);
    if (st != MOE_OK)
        return done(st);
    return launched(moe::combine_fp8(y_q, y_scale, dispatch_pos, topk_w, T, H, k, rows, out,
                                     dev_status, as_stream(stream)));
}

// Shared experts and replicas for the fused launch: the same checks as
// moe_route_topk_ex; the replica choice uses T / R tokens per source rank.
static int route_dispatch_ex(const float *logits, int T, int E, int k, int renormalize,
                             int n_shared, float shared_weight, const int32_t *replica_offsets,
                             const int32_t *replica_ids, int n_replica_ids, int E_phys, int R,
                             int capacity, const uint16_t *x, int H, bool fp8, int32_t *topk_idx,
                             float *topk_w, int32_t *expert_counts, int32_t *expert_src_counts,
                             int32_t *rank_counts, int32_t *expert_offsets, int32_t *dispatch_pos,
                             int32_t *recv_src, void *recv, float *recv_scale, int64_t rows,
                             void *workspace, size_t ws_bytes, int32_t *dev_status, void *stream)
{
    if (n_shared < 0 || n_shared > kMaxK || k < 1 || k + n_shared > kMaxK || E < 1 || E > kMaxE ||
        E_phys < 1 || E_phys > kMaxE || R < 1)
        return MOE_ERR_INVALID_ARG;
    if (replica_offsets != nullptr &&
        (replica_ids == nullptr || n_replica_ids < 1 || !aligned(replica_offsets, 4) ||
         !aligned(replica_ids, 4)))
        return MOE_ERR_INVALID_ARG;
    if (replica_offsets == nullptr && E_phys < E + n_shared)
        return MOE_ERR_INVALID_ARG;
    const int tpr = (T >= R && T % R == 0) ? T / R : 1;
    const moe::RouteEx ex{n_shared, shared_weight, replica_offsets, replica_ids, n_replica_ids,
                          E_phys, tpr, dev_status};
    return route_dispatch_common(logits, T, E, k, renormalize, R, capacity, x, H, fp8, topk_idx,
                                 topk_w, expert_counts, expert_src_counts, rank_counts,
                                 expert_offsets, dispatch_pos, recv_src, recv, recv_scale, rows,
                                 workspace, ws_bytes, dev_status, stream, &ex);
}

int moe_route_dispatch_ex_fp8(const float *logits, int T, int E, int k, int renormalize,
                              int n_shared, float shared_weight, const int32_t *replica_offsets,
                              const int32_t *replica_ids, int n_replica_ids, int E_phys, int R,
                              int capacity, const uint16_t *x, int H, int32_t *topk_idx,
                              float *topk_w, int32_t *expert_counts, int32_t *expert_src_counts,
                              int32_t *rank_counts, int32_t *expert_offsets, int32_t *dispatch_pos,
                              int32_t *recv_src, uint8_t *recv_q, float *recv_scale, int64_t rows,
                              void *workspace, size_t ws_bytes, int32_t *dev_status, void *stream)
{
    return route_dispatch_ex(logits, T, E, k, renormalize, n_shared, shared_weight,
                             replica_offsets, replica_ids, n_replica_ids, E_phys, R, capacity, x, H,
                             true, topk_idx, topk_w, expert_counts, expert_src_counts, rank_counts,
                             expert_offsets, dispatch_pos, recv_src, recv_q, recv_scale, rows,
                             workspace, ws_bytes, dev_status, stream);
}

int moe_route_dispatch_ex_bf16(const float *logits, int T, int E, int k, int renormalize,
                               int n_shared, float shared_weight, const int32_t *replica_offsets,
                               const int32_t *replica_ids, int n_replica_ids, int E_phys, int R,
                               int capacity, const uint16_t *x, int H, int32_t *topk_idx,
                               float *topk_w, int32_t *expert_counts, int32_t *expert_src_counts,
                               int32_t *rank_counts, int32_t *expert_offsets,
                               int32_t *dispatch_pos, int32_t *recv_src, uint16_t *recv_x,
                               int64_t rows, void *workspace, size_t ws_bytes, int32_t *dev_status,
                               void *stream)
{
    return route_dispatch_ex(logits, T, E, k, renormalize, n_shared, shared_weight,
                             replica_offsets, replica_ids, n_replica_ids, E_phys, R, capacity, x, H,
                             false, topk_idx, topk_w, expert_counts, expert_src_counts, rank_counts,
                             expert_offsets, dispatch_pos, recv_src, recv_x, nullptr, rows,
                             workspace, ws_bytes, dev_status, stream);
}

// ---- host-buffer entry points: the copies, then the same launches ----------

static int copy_async(void *dst, const void *src, size_t bytes, cudaMemcpyKind kind,
                      cudaStream_t s)
{
    return bytes == 0 ? MOE_OK : launched(cudaMemcpyAsync(dst, src, bytes, kind, s));
}

static int route_dispatch_host(const float *logits_host, const uint16_t *x_host, int T, int E,
                               int k, int renormalize, int R, int capacity, int H, bool fp8,
                               int flags, float *logits, uint16_t *x, int32_t *topk_idx,
                               float *topk_w, int32_t *expert_counts, int32_t *expert_src_counts,
                               int32_t *rank_counts, int32_t *expert_offsets,
                               int32_t *dispatch_pos, int32_t *recv_src, void *recv,
                               float *recv_scale, int64_t rows, void *workspace, size_t ws_bytes,
                               int32_t *dev_status, void *stream)
{
    if ((flags & ~MOE_HOST_FUSED) != 0)
        return MOE_ERR_INVALID_ARG;
    const bool fused = (flags & MOE_HOST_FUSED) != 0;
    int st;
    if (fused) {
        st = route_dispatch_args(logits, T, E, k, R, capacity, x, H, fp8, topk_idx, topk_w,
                                 expert_counts, expert_src_counts, rank_counts, expert_offsets,
                                 dispatch_pos, recv_src, recv, recv_scale, rows, workspace,
                                 dev_status, nullptr);
        if (st == MOE_OK && ws_bytes < moe::route_dispatch_workspace_bytes(T, k, E, R))
            st = MOE_ERR_WORKSPACE;
    } else {
        st = done(route_topk_args(logits, T, E, k, topk_idx, topk_w));
        if (st == MOE_OK)
            st = layout_args(topk_idx, T, k, E, R, capacity, rows, expert_counts,
                             expert_src_counts, rank_counts, expert_offsets, dispatch_pos,
                             recv_src, workspace, ws_bytes, dev_status);
        if (st == MOE_OK)
            st = done(fp8 ? dispatch_fp8_args(x, T, H, k, dispatch_pos,
                                              static_cast<const uint8_t *>(recv), recv_scale, rows,
                                              dev_status)
                          : dispatch_bf16_args(x, T, H, k, dispatch_pos,
                                               static_cast<const uint16_t *>(recv), rows,
                                               dev_status));
    }
    if (st != MOE_OK)
        return st;
    if (T > 0 && (!logits_host || !x_host))
        return MOE_ERR_INVALID_ARG;

    const cudaStream_t s = as_stream(stream);
    // T * E fp32 and T * H bf16: E <= 1024 and H checked above
    st = copy_async(logits, logits_host, static_cast<size_t>(T) * E * sizeof(float),
                    cudaMemcpyHostToDevice, s);
    if (st == MOE_OK)
        st = copy_async(x, x_host, static_cast<size_t>(T) * H * sizeof(uint16_t),
                        cudaMemcpyHostToDevice, s);
    if (st != MOE_OK)
        return st;
    if (fused) {
        bool small = false;
        const cudaError_t err = moe::route_dispatch(
            logits, T, E, k, renormalize != 0, R, capacity, x, H, fp8, topk_idx, topk_w,
            expert_counts, expert_src_counts, rank_counts, expert_offsets, dispatch_pos, recv_src,
            recv, recv_scale, rows, workspace, ws_bytes, dev_status, s, &small, nullptr);
        return small ? MOE_ERR_WORKSPACE : launched(err);
    }
    if (T > 0) {
        st = launched(moe::route_topk(logits, T, E, k, renormalize != 0, topk_idx, topk_w,
                                      nullptr, s));
        if (st != MOE_OK)
            return st;
    }
    st = launched(moe::dispatch_layout(topk_idx, moe::layout_geom(T, k, E, R), capacity, rows,
                                       expert_counts, expert_src_counts, rank_counts,
                                       expert_offsets, dispatch_pos, recv_src, nullptr,
                                       workspace, dev_status, s));
    if (st != MOE_OK || T == 0)
        return st;
    return launched(fp8 ? moe::dispatch_fp8(x, T, H, k, dispatch_pos, static_cast<uint8_t *>(recv),
                                            recv_scale, rows, 0, dev_status, s)
                        : moe::dispatch_bf16(x, T, H, k, dispatch_pos,
                                             static_cast<uint16_t *>(recv), rows, dev_status, s));
}

int moe_route_dispatch_fp8_host(const float *logits_host, const uint16_t *x_host, int T, int E,
                                int k, int renormalize, int R, int capacity, int H, int flags,
                                float *logits, uint16_t *x, int32_t *topk_idx, float *topk_w,
                                int32_t *expert_counts, int32_t *expert_src_counts,
                                int32_t *rank_counts, int32_t *expert_offsets,
                                int32_t *dispatch_pos, int32_t *recv_src, uint8_t *recv_q,
                                float *recv_scale, int64_t rows, void *workspace, size_t ws_bytes,
                                int32_t *dev_status, void *stream)
{
    return route_dispatch_host(logits_host, x_host, T, E, k, renormalize, R, capacity, H, true,
                               flags, logits, x, topk_idx, topk_w, expert_counts,
                               expert_src_counts, rank_counts, expert_offsets, dispatch_pos,
                               recv_src, recv_q, recv_scale, rows, workspace, ws_bytes, dev_status,
                               stream);
}

int moe_route_dispatch_bf16_host(const float *logits_host, const uint16_t *x_host, int T, int E,
                                 int k, int renormalize, int R, int capacity, int H, int flags,
                                 float *logits, uint16_t *x, int32_t *topk_idx, float *topk_w,
                                 int32_t *expert_counts, int32_t *expert_src_counts,
                                 int32_t *rank_counts, int32_t *expert_offsets,
                                 int32_t *dispatch_pos, int32_t *recv_src, uint16_t *recv_x,
                                 int64_t rows, void *workspace, size_t ws_bytes,
                                 int32_t *dev_status, void *stream)
{
    return route_dispatch_host(logits_host, x_host, T, E, k, renormalize, R, capacity, H, false,
                               flags, logits, x, topk_idx, topk_w, expert_counts,
                               expert_src_counts, rank_counts, expert_offsets, dispatch_pos,
                               recv_src, recv_x, nullptr, rows, workspace, ws_bytes, dev_status,
                               stream);
}

int moe_combine_bf16_host(const uint16_t *y, const int32_t *dispatch_pos, const float *topk_w,
                          int T, int H, int k, int64_t rows, uint16_t *out, uint16_t *out_host,
                          int32_t *dev_status, void *stream)
{
    const int st = combine_bf16_args(y, dispatch_pos, topk_w, T, H, k, rows, out, dev_status);
    if (st != MOE_OK)
        return done(st);
    if (!out_host)
        return MOE_ERR_INVALID_ARG;
    const cudaStream_t s = as_stream(stream);
    const int lst = launched(moe::combine_bf16(y, dispatch_pos, topk_w, T, H, k, rows, out,
                                               dev_status, s));
    if (lst != MOE_OK)
        return lst;
    return copy_async(out_host, out, static_cast<size_t>(T) * H * sizeof(uint16_t),
                      cudaMemcpyDeviceToHost, s);
}

int moe_combine_fp8_host(const uint8_t *y_q, const float *y_scale, const int32_t *dispatch_pos,
                         const float *topk_w, int T, int H, int k, int64_t rows, uint16_t *out,
                         uint16_t *out_host, int32_t *dev_status, void *stream)
{
    const int st = combine_fp8_args(y_q, y_scale, dispatch_pos, topk_w, T, H, k, rows, out,
                                    dev_status);
    if (st != MOE_OK)
        return done(st);
    if (!out_host)
        return MOE_ERR_INVALID_ARG;
    const cudaStream_t s = as_stream(stream);
    const int lst = launched(moe::combine_fp8(y_q, y_scale, dispatch_pos, topk_w, T, H, k, rows,
                                              out, dev_status, s));
    if (lst != MOE_OK)
        return lst;
    return copy_async(out_host, out, static_cast<size_t>(T) * H * sizeof(uint16_t),
                      cudaMemcpyDeviceToHost, s);
}

int moe_quantize_e4m3(const float *v, int64_t n, uint8_t *q, void *stream)
{
    if (n < 0)
        return MOE_ERR_INVALID_ARG;
    if (n == 0)
        return MOE_OK;
    if (!v || !q || !aligned(v, 4))
        return MOE_ERR_INVALID_ARG;
    return launched(moe::quantize_e4m3(v, n, q, as_stream(stream)));
}

}  // extern "C"
