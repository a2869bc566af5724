// kernels.cuh -- launchers of the libmoe_route kernels (internal to the
// library; the public surface is include/moe_route.h).  Arguments arrive here
// already validated by the C ABI layer.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

// Layout geometry: tokens are cut into chunks that never straddle two logical
// source ranks; one CTA counts, and later places, the slots of one chunk.
struct LayoutGeom {
    int T, k, E, R;
    int Tr;       // tokens per logical source rank
    int CT;       // tokens per chunk
    int cpr;      // chunks per rank
    int nchunks;  // R * cpr
    int max_m;    // > 0: also place every slot in its private (expert, source rank) region
};

LayoutGeom layout_geom(int T, int k, int E, int R);
size_t layout_workspace_bytes(const LayoutGeom &g);
// Kernels dispatch_layout launches for g on the current device (1 or 2).
int layout_launches(const LayoutGeom &g);

// Extension of the route: shared experts and expert replicas.
struct RouteEx {
    int n_shared;
    float shared_weight;
    const int32_t *replica_offsets;  // [E + n_shared + 1] or nullptr
    const int32_t *replica_ids;      // [n_replica_ids]
    int n_replica_ids;
    int E_phys;
    int tokens_per_rank;
    int32_t *dev_status;
};

// ex == nullptr: the plain route (outputs [T][k]); otherwise outputs are
// [T][k + ex->n_shared] physical expert ids.
cudaError_t route_topk(const float *logits, int T, int E, int k, int renormalize,
                       int32_t *topk_idx, float *topk_w, const RouteEx *ex, cudaStream_t s);

// private_pos: [T][k] private rows when g.max_m > 0 (else unused, may be null).
cudaError_t dispatch_layout(const int32_t *topk_idx, const LayoutGeom &g, int capacity,
                            int64_t rows, int32_t *expert_counts, int32_t *expert_src_counts,
                            int32_t *rank_counts, int32_t *expert_offsets,
                            int32_t *dispatch_pos, int32_t *recv_src, int32_t *private_pos,
                            void *workspace, int32_t *dev_status, cudaStream_t s);

// Receiver side of the two-phase dispatch: copy every slot's private row to
// its packed row (codes and scales / bf16 rows).
cudaError_t compact_fp8(const uint8_t *priv_q, const float *priv_scale, int64_t private_rows,
                        const int32_t *private_pos, const int32_t *dispatch_pos, int T, int H,
                        int k, uint8_t *recv_q, float *recv_scale, int64_t rows,
                        int32_t *dev_status, cudaStream_t s);
cudaError_t compact_bf16(const uint16_t *priv_x, int64_t private_rows, const int32_t *private_pos,
                         const int32_t *dispatch_pos, int T, int H, int k, uint16_t *recv_x,
                         int64_t rows, int32_t *dev_status, cudaStream_t s);

cudaError_t dispatch_bf16(const uint16_t *x, int T, int H, int k, const int32_t *dispatch_pos,
                          uint16_t *recv_x, int64_t rows, int32_t *dev_status, cudaStream_t s);

// scale_ld == 0: scales row-major [rows][H/128]; > 0: column-major
// [H/128][scale_ld] (scale_ld >= rows).
cudaError_t dispatch_fp8(const uint16_t *x, int T, int H, int k, const int32_t *dispatch_pos,
                         uint8_t *recv_q, float *recv_scale, int64_t rows, int64_t scale_ld,
                         int32_t *dev_status, cudaStream_t s);

cudaError_t combine_bf16(const uint16_t *y, const int32_t *dispatch_pos, const float *topk_w,
                         int T, int H, int k, int64_t rows, uint16_t *out, int32_t *dev_status,
                         cudaStream_t s);
// Whether combine_bf16 takes its long, 32-byte-load form for these sizes when
// y and out are 32-byte aligned.
bool combine_bf16_long_form(int T, int H, int k);

// Route + layout + dispatch in one cooperative launch (packed or padded
// layout).  E, k: the router's experts and routed slots; with ex the layout
// sees k + ex->n_shared slots over ex->E_phys experts, as after
// route_topk(..., ex).  Workspace bytes depend on the current device's SM
// count (0 = no device); they are given for the layout's (k, E).
// *ws_too_small is set (and nothing launched) when ws_bytes is below what the
// geometry needs.
size_t route_dispatch_workspace_bytes(int T, int k, int E, int R);
cudaError_t route_dispatch(const float *logits, int T, int E, int k, int renormalize, int R,
                           int capacity, const uint16_t *x, int H, bool fp8, int32_t *topk_idx,
                           float *topk_w, int32_t *expert_counts, int32_t *expert_src_counts,
                           int32_t *rank_counts, int32_t *expert_offsets, int32_t *dispatch_pos,
                           int32_t *recv_src, void *recv, float *recv_scale, int64_t rows,
                           void *workspace, size_t ws_bytes, int32_t *dev_status, cudaStream_t s,
                           bool *ws_too_small, const RouteEx *ex = nullptr);

// Combine with E4M3 rows yq [rows][H] and row-major 1x128 scales ys [rows][H/128].
cudaError_t combine_fp8(const uint8_t *yq, const float *ys, const int32_t *dispatch_pos,
                        const float *topk_w, int T, int H, int k, int64_t rows, uint16_t *out,
                        int32_t *dev_status, cudaStream_t s);

cudaError_t quantize_e4m3(const float *v, int64_t n, uint8_t *q, cudaStream_t s);

// How many bytes of x (x_bytes = T*H*2) a dispatch prefetches into L2 ahead of
// its wait, and from how many CTAs (0 bytes when x would not fit in L2).
void prefetch_plan(int64_t x_bytes, int64_t &pf_bytes, int &pf_ctas);

}  // namespace moe
