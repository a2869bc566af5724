/*
 * moe_route.h -- C ABI of libmoe_route.so: Mixture-of-Experts routing,
 * dispatch and combine on one GPU (sm_100a).
 *
 * The path: router logits -> softmax + top-k (moe_route_topk) -> per-expert
 * counts, offsets and index maps (moe_dispatch_layout) -> row scatter of each
 * token into per-expert receive buffers, as bf16 or as e4m3 with 1x128 block
 * scales (moe_dispatch_bf16 / moe_dispatch_fp8) -> [expert computation, not
 * part of this library] -> gather of the expert outputs and the router-
 * weighted sum per token (moe_combine_bf16).  Expert-parallel ranks are
 * logical: R partitions of this one device's memory.  Nothing here talks to
 * another GPU.
 *
 * Sources (page title, section):
 *   "Efficient and portable mixture-of-experts communication" (Perplexity,
 *     2025-04-02): "Introdução", "Despacho", "Combinação".
 *   "Enabling trillion-parameter models on AWS EFA" (Perplexity, 2025-11-04):
 *     "Gönderme ve Alma Arabellekleri", "Dağıtım ve Birleştirme",
 *     "Dağıtım/Birleştirme Gecikmesi".
 *   DeepSeek-V3 report fragments quoted on the other pages: 1x128 activation
 *     tiles (per token per 128 channels), gating kept in original precision,
 *     combine kept in BF16.
 *
 * Conventions shared by every entry point
 *   - Every array pointer is a DEVICE pointer owned by the caller, except
 *     the *_host arguments of the host-buffer entry points (near the end of
 *     this file).  The library allocates nothing, keeps no pointer after the
 *     call returns and never synchronises the device.
 *   - bf16 data are passed as their 16-bit patterns (uint16_t).
 *   - `stream` is a cudaStream_t (CUstream) passed as void*; NULL is the
 *     legacy default stream.  All device work is enqueued on it and runs
 *     asynchronously.
 *   - Argument errors are detected on the host before anything is enqueued
 *     and returned synchronously (MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED).
 *     A failed launch returns MOE_ERR_CUDA.
 *   - Errors found by the kernels themselves (an expert id or row outside its
 *     range, a capacity overflow) are written to *dev_status, an int32 in
 *     device memory that the caller zeroes beforehand and reads after the
 *     stream has been synchronised: the first error code written wins.  A
 *     kernel that finds such an error skips the offending element; it never
 *     traps and never touches memory outside the documented ranges.
 *     dev_status may be NULL (errors are then skipped silently).
 *   - Row data pointers (x, recv_x, recv_q, y, out) must be 16-byte aligned;
 *     recv_scale, logits and the index arrays 4-byte aligned.
 *   - Sizes: 0 <= T, 1 <= k <= min(E, 32), 1 <= E <= 1024, 1 <= R <= E,
 *     E % R == 0, T % R == 0 (T/R tokens per logical source rank), H % 8 == 0
 *     (bf16 paths), H % 128 == 0 (fp8 path), T*k < 2^31, rows < 2^31.
 *
 * Token g = r*(T/R) + t belongs to logical source rank r; expert e lives on
 * logical destination rank e / (E/R).  Slot i = g*k + j is token g's j-th
 * expert choice.
 */
#ifndef MOE_ROUTE_H
#define MOE_ROUTE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* bad size, NULL or misaligned pointer, bad id/row */
    MOE_ERR_UNSUPPORTED = 2, /* valid request the library does not support (fp8 with H % 128 != 0) */
    MOE_ERR_CAPACITY = 3,    /* padded layout: a slot beyond its expert's capacity was dropped */
    MOE_ERR_WORKSPACE = 4,   /* workspace too small or misaligned */
    MOE_ERR_TIMEOUT = 5,     /* a bounded wait inside a kernel gave up */
    MOE_ERR_CUDA = 6         /* a CUDA launch or runtime call failed */
} moe_status_t;

/* Human-readable name of a status code (static string, never NULL). */
const char *moe_status_string(int status);

/*
 * moe_route_topk -- router softmax and top-k selection.
 * Follows "Efficient and portable mixture-of-experts communication",
 * "Introdução": the router's small linear layer yields a probability
 * distribution over experts; the top-K experts are chosen and each expert
 * output is weighted by a weight derived from that distribution.  Gating stays
 * in its original precision (DeepSeek-V3 fragments): fp32 in, fp32 out.
 *
 *   logits    [T][E] fp32, row-major (E contiguous).
 *   topk_idx  [T][k] int32 out: the k experts first in the order (logit
 *             descending, expert index ascending); -0.0 and +0.0 are equal.
 *   topk_w    [T][k] fp32 out: p_e = exp(l_e - m) / sum_e' exp(l_e' - m),
 *             m = max logit; with renormalize != 0 the sum runs over the k
 *             chosen experts only (softmax restricted to the top-k).  Terms in
 *             fp32 (exact split of l - m, expf), their sum in binary64 rounded
 *             once, one IEEE division: |topk_w - p| <= 7 * 2^-24 * p.
 * Logits must be finite.  T == 0 enqueues nothing.
 */
int moe_route_topk(const float *logits, int T, int E, int k, int renormalize,
                   int32_t *topk_idx, float *topk_w, void *stream);

/*
 * moe_route_topk_ex -- moe_route_topk with shared experts and expert replicas.
 * Follows the DeepSeek-V3 report fragments quoted on the third and fourth
 * pages: during decoding the shared expert is treated as a routed one that
 * every token always selects (so each token selects 9 experts), and each GPU
 * also hosts redundant replicas of heavily loaded experts.
 *
 *   Routed part: exactly moe_route_topk over the E routed logits (k experts,
 *   weights as there, renormalize over the k routed ones).  Shared part: the
 *   n_shared logical experts E .. E + n_shared - 1 follow in slot order, each
 *   with weight shared_weight.  Every chosen logical expert l is mapped to a
 *   physical expert:
 *     replica_offsets == NULL: physical id = l (needs E_phys >= E + n_shared);
 *     otherwise l is served by replica_ids[replica_offsets[l] ..
 *     replica_offsets[l + 1]) and the token g of source rank
 *     r = g / tokens_per_rank uses replica r mod (number of replicas of l).
 *   replica_offsets  [E + n_shared + 1] int32 (device), non-decreasing.
 *   replica_ids      [n_replica_ids] int32 (device) physical ids in [0, E_phys).
 *   topk_idx         [T][k + n_shared] int32 out: physical expert ids.
 *   topk_w           [T][k + n_shared] fp32 out.
 * A slot whose table entry is empty, out of [0, n_replica_ids) or gives an id
 * outside [0, E_phys) gets -1 and MOE_ERR_INVALID_ARG through dev_status.
 * Limits: 0 <= n_shared, 1 <= k, k + n_shared <= 32, tokens_per_rank >= 1.
 * The output feeds moe_dispatch_layout with E_phys experts.
 */
int moe_route_topk_ex(const float *logits, int T, int E, int k, int renormalize, int n_shared,
                      float shared_weight, const int32_t *replica_offsets,
                      const int32_t *replica_ids, int n_replica_ids, int E_phys,
                      int tokens_per_rank, int32_t *topk_idx, float *topk_w, int32_t *dev_status,
                      void *stream);

/*
 * Bytes of device workspace moe_dispatch_layout needs for (T, k, E, R);
 * 0 on invalid sizes.  The workspace must be 256-byte aligned; its contents
 * need no initialisation and are scratch (per-chunk histograms).  One
 * workspace must not serve two layout calls that may run at the same time.
 */
size_t moe_layout_workspace_bytes(int T, int k, int E, int R);

/*
 * How many kernels moe_dispatch_layout (and moe_dispatch_layout_private)
 * launch for (T, k, E, R) on the current device: 1 for small layouts, when
 * every logical rank fits one chunk of at most 2048 slots, the slots come to
 * at most one per thread of an 8-CTA cluster of 1024 threads each (T*k <=
 * 8192) and the device can schedule that cluster; else 2 (a per-chunk
 * histogram, then the placement).  0 on invalid sizes.  Both forms give identical outputs; the
 * count serves callers that account for launches (graph sizing, profiling).
 */
int moe_dispatch_layout_launches(int T, int k, int E, int R);

/*
 * moe_dispatch_layout -- counts, offsets and index maps for dispatch/combine.
 * Follows "Enabling trillion-parameter models on AWS EFA", "Gönderme ve Alma
 * Arabellekleri" (per-expert token counts first; then every sender knows
 * where its writes go; receive buffers are contiguous) and "Dağıtım ve
 * Birleştirme" (counts per expert, cumulative sums -> offsets that pack tokens
 * into contiguous per-expert buffers); "Efficient and portable mixture-of-
 * experts communication", "Despacho" (source rank, expert index and token
 * index kept for combine; tokens grouped per expert).
 *
 *   topk_idx          [T][k] int32: expert of each slot.  -1 marks an empty
 *                     slot (skipped, not counted); any other id outside
 *                     [0, E) is skipped and reported as MOE_ERR_INVALID_ARG
 *                     through dev_status.
 *   capacity          0: packed.  Expert e owns rows [off_e, off_e + n_e),
 *                     off = exclusive prefix sum of the counts in expert
 *                     order, so logical rank r's region is the contiguous
 *                     run of its experts [r*E/R, (r+1)*E/R).
 *                     > 0: padded.  Expert e owns rows [e*cap, (e+1)*cap); a
 *                     slot at position >= cap inside its expert is dropped
 *                     (dispatch_pos = -1) and MOE_ERR_CAPACITY is reported
 *                     through dev_status.
 *   rows              length of recv_src; at least T*k (packed) or E*cap
 *                     (padded).
 *   Slots of one expert take consecutive rows in ascending slot index
 *   i = g*k + j (ascending source rank, then token): the layout is
 *   deterministic.
 *   expert_counts     [E]    out: slots routed to e (dropped ones included).
 *   expert_src_counts [E][R] out: slots routed to e from source rank r.
 *   rank_counts       [R]    out: slots routed to rank r's experts.
 *   expert_offsets    [E+1]  out: first row of expert e; [E] = packed total
 *                     or E*cap.
 *   dispatch_pos      [T][k] out: row of slot (g, j), or -1.
 *   recv_src          [rows] out: the slot i = g*k + j a row holds, or -1
 *                     for every row no slot fills.
 *   workspace         see moe_layout_workspace_bytes; MOE_ERR_WORKSPACE if
 *                     ws_bytes is too small or the pointer misaligned.
 */
int moe_dispatch_layout(const int32_t *topk_idx, int T, int k, int E, int R,
                        int capacity, int64_t rows, int32_t *expert_counts,
                        int32_t *expert_src_counts, int32_t *rank_counts,
                        int32_t *expert_offsets, int32_t *dispatch_pos,
                        int32_t *recv_src, void *workspace, size_t ws_bytes,
                        int32_t *dev_status, void *stream);

/*
 * Two-phase dispatch (the pages' own design, for comparison with the direct
 * scatter above).  "Efficient and portable mixture-of-experts
 * communication", "Kernels portáteis": each rank keeps private storage to
 * receive from every other rank; the number of tokens a source rank may
 * dispatch is fixed, which bounds what a rank receives for each local expert
 * from each source rank, so senders derive unique addresses without
 * synchronising; after receiving, the tokens are reorganised into the layout
 * the expert kernels need ("Despacho": copied into contiguous buffers).
 *
 * moe_dispatch_layout_private -- everything moe_dispatch_layout (packed,
 * capacity 0) outputs, identically, plus
 *   private_pos [T][k] int32 out: the slot's row in the private region of
 *               (its expert e, its source rank r): rows
 *               [(e*R + r)*max_m, (e*R + r + 1)*max_m), position = number of
 *               earlier slots of the same source rank routed to e.  A slot at
 *               position >= max_m is dropped: private_pos and dispatch_pos -1,
 *               its packed row left empty (recv_src -1), MOE_ERR_CAPACITY
 *               through dev_status.  max_m = T/R never drops (a token picks an
 *               expert at most once).
 * The private rows hold E*R*max_m rows (< 2^31).  Send phase: moe_dispatch_fp8
 * (or _bf16) with private_pos as dispatch_pos and rows = E*R*max_m.
 */
int moe_dispatch_layout_private(const int32_t *topk_idx, int T, int k, int E, int R, int max_m,
                                int64_t rows, int32_t *expert_counts, int32_t *expert_src_counts,
                                int32_t *rank_counts, int32_t *expert_offsets,
                                int32_t *dispatch_pos, int32_t *recv_src, int32_t *private_pos,
                                void *workspace, size_t ws_bytes, int32_t *dev_status,
                                void *stream);

/*
 * moe_compact_fp8 / moe_compact_bf16 -- receive phase of the two-phase
 * dispatch: for every slot with private_pos >= 0, copy its private row
 * (codes and 1x128 scales, or bf16 row) to row dispatch_pos of the packed
 * buffers.  The result is byte-for-byte what moe_dispatch_fp8 / _bf16 write
 * with dispatch_pos directly.  A row outside [0, private_rows) or [0, rows)
 * is skipped and reported (MOE_ERR_INVALID_ARG via dev_status).
 *   priv_q [private_rows][H] u8, priv_scale [private_rows][H/128] fp32 (or
 *   priv_x [private_rows][H] bf16) -> recv_q / recv_scale (recv_x) [rows][...].
 */
int moe_compact_fp8(const uint8_t *priv_q, const float *priv_scale, int64_t private_rows,
                    const int32_t *private_pos, const int32_t *dispatch_pos, int T, int H, int k,
                    uint8_t *recv_q, float *recv_scale, int64_t rows, int32_t *dev_status,
                    void *stream);
int moe_compact_bf16(const uint16_t *priv_x, int64_t private_rows, const int32_t *private_pos,
                     const int32_t *dispatch_pos, int T, int H, int k, uint16_t *recv_x,
                     int64_t rows, int32_t *dev_status, void *stream);

/*
 * moe_dispatch_layout_noalloc -- moe_dispatch_layout for callers that cannot
 * allocate device memory.  The pages have no counterpart: this is a
 * deployment variant of the entry point above, not a step of the method.
 *
 * Some callers cannot hand the layout a workspace: a plugin or custom-op
 * layer that receives only its input and output buffers and no allocator,
 * a host callback or latency-critical loop where cudaMalloc would
 * synchronise the device, a deployment whose device memory is budgeted up
 * front.  This entry point takes the same arguments as moe_dispatch_layout
 * minus the workspace, and allocates nothing (no cudaMalloc, no cudaFree,
 * no allocating library call).  Its scratch is a file-scope __device__
 * array of MOE_LAYOUT_NOALLOC_SCRATCH_BYTES (1 MiB) inside this library:
 * every GPU that loads the library holds it until the process exits.
 *
 *   - Limit: a call fits exactly when moe_layout_workspace_bytes(T, k, E, R)
 *     <= MOE_LAYOUT_NOALLOC_SCRATCH_BYTES; larger sizes are rejected with
 *     MOE_ERR_WORKSPACE before anything is enqueued.  That size is
 *     max(256, round_up(R * ceil((T/R) / max(1, floor(2048/k))) * E * 4, 256))
 *     bytes: one E-wide int32 histogram row per chunk, where a chunk is at
 *     most floor(2048/k) tokens of one logical rank, so a partly filled chunk
 *     still takes a whole row.  (E = 256, k = 8: up to 1024 chunks, e.g.
 *     T/R = 256 tokens per rank and R <= 1024; every workload of the
 *     benchmark fits.)
 *   - Set-up: the first call on each device looks the array's device address
 *     up (cudaGetSymbolAddress, with that device current); every later call
 *     made outside stream capture looks it up again (a host query, no
 *     allocation), so a device reset or a re-created context never leaves a
 *     stale address.  Calls during stream capture reuse the last address
 *     found outside capture: make the first call on each device before any
 *     stream capture on it, else the call returns MOE_ERR_UNSUPPORTED.  Any
 *     number of devices is served (the table is sized from
 *     cudaGetDeviceCount).
 *   - Sharing: all calls share the one array and it keeps the last call's
 *     contents.  Each call rewrites every scratch word it reads, so nothing
 *     needs clearing, but two calls whose kernels overlap on the GPU (other
 *     streams, other host threads) race on the array: serialise them.
 *   - Arguments, outputs and errors are otherwise those of
 *     moe_dispatch_layout.
 */
#define MOE_LAYOUT_NOALLOC_SCRATCH_BYTES ((size_t)1 << 20)

int moe_dispatch_layout_noalloc(const int32_t *topk_idx, int T, int k, int E, int R,
                                int capacity, int64_t rows, int32_t *expert_counts,
                                int32_t *expert_src_counts, int32_t *rank_counts,
                                int32_t *expert_offsets, int32_t *dispatch_pos,
                                int32_t *recv_src, int32_t *dev_status, void *stream);

/*
 * moe_dispatch_bf16 -- row scatter: recv_x[dispatch_pos[g][j]] = x[g].
 * Follows "Enabling trillion-parameter models on AWS EFA", "Dağıtım ve
 * Birleştirme" (tokens packed into contiguous per-expert buffers) and
 * "Efficient and portable mixture-of-experts communication", "Despacho".
 *
 *   x             [T][H] bf16 bits, row-major.
 *   dispatch_pos  [T][k] int32 rows from moe_dispatch_layout; -1 skipped; a
 *                 row outside [0, rows) is skipped and reported
 *                 (MOE_ERR_INVALID_ARG via dev_status).
 *   recv_x        [rows][H] bf16 bits out; rows no slot targets are not
 *                 written.
 * T == 0 enqueues nothing.  When x fits in three quarters of L2, the kernel's
 * first CTAs issue L2 prefetches of x before they wait for the kernel ahead
 * of them on the stream (a scheduling hint: no effect on any result).
 */
int moe_dispatch_bf16(const uint16_t *x, int T, int H, int k,
                      const int32_t *dispatch_pos, uint16_t *recv_x,
                      int64_t rows, int32_t *dev_status, void *stream);

/*
 * moe_dispatch_fp8 -- quantise each token once on 1x128 blocks and scatter
 * the codes and scales to its k rows.
 * Follows "Enabling trillion-parameter models on AWS EFA", "Dağıtım/
 * Birleştirme Gecikmesi" (block-scaled fp8 dispatch) and the DeepSeek-V3
 * fragments (activations scaled per token per 128 channels); the format is
 * OCP E4M3 (max finite 448).
 *
 *   For each token g and block b of 128 channels:
 *     amax = max |x|, s = amax / 448 (IEEE binary32 division; s = 1 when
 *     amax == 0), q = e4m3(x / s) (binary32 division, round to nearest even,
 *     saturating at +-448).
 *   recv_q      [rows][H] uint8 e4m3 codes out.
 *   recv_scale  [rows][H/128] fp32 scales out (dequantised value = e4m3(q)*s).
 *   dispatch_pos, rows, dev_status: as for moe_dispatch_bf16 (L2 prefetch of
 *   x included).
 * Performance note: when x is too large to be prefetched into L2 (more than
 * three quarters of it), H % 256 == 0 and recv_q is 32-byte aligned, each
 * thread quantises 32 channels and writes them with one 32-byte store; the
 * codes and scales are the same either way.
 * H % 128 != 0 returns MOE_ERR_UNSUPPORTED.  T == 0 enqueues nothing.
 */
int moe_dispatch_fp8(const uint16_t *x, int T, int H, int k,
                     const int32_t *dispatch_pos, uint8_t *recv_q,
                     float *recv_scale, int64_t rows, int32_t *dev_status,
                     void *stream);

/*
 * moe_dispatch_fp8_ex -- moe_dispatch_fp8 with a choice of scale layout for
 * the grouped GEMM that consumes the rows.  The codes, the scale values and
 * the rows written are exactly those of moe_dispatch_fp8 (DeepSeek-V3
 * fragments: 1x128 activation tiles); only where each scale is stored
 * changes.
 *   scale_layout MOE_SCALE_ROW_MAJOR: recv_scale [rows][H/128] (scale_ld
 *                ignored), as moe_dispatch_fp8.
 *   scale_layout MOE_SCALE_COL_MAJOR: recv_scale [H/128][scale_ld], the scale
 *                of row r and block b at recv_scale[b * scale_ld + r];
 *                scale_ld >= rows and scale_ld % 4 == 0 so every block's
 *                column starts 16-byte aligned (recv_scale itself 16-byte
 *                aligned), the layout a tile load along the rows needs.
 *                Entries of rows no slot fills are not written.
 */
#define MOE_SCALE_ROW_MAJOR 0
#define MOE_SCALE_COL_MAJOR 1

int moe_dispatch_fp8_ex(const uint16_t *x, int T, int H, int k, const int32_t *dispatch_pos,
                        uint8_t *recv_q, float *recv_scale, int64_t rows, int scale_layout,
                        int64_t scale_ld, int32_t *dev_status, void *stream);

/*
 * moe_route_dispatch_fp8 / moe_route_dispatch_bf16 -- moe_route_topk,
 * moe_dispatch_layout and moe_dispatch_fp8 (or _bf16) in ONE launch.
 * Follows "Enabling trillion-parameter models on AWS EFA", "Dağıtım ve
 * Birleştirme" (the dispatch kernel counts the tokens of each expert itself,
 * by atomic accumulation in shared memory within a block, sums the counts
 * into offsets and packs the tokens at those offsets) and "Efficient and
 * portable mixture-of-experts communication", "Despacho" (one routing warp
 * counts while the others move the tokens).
 *
 * Outputs are bit-identical to the three separate calls with the same
 * arguments (plain route, scales row-major):
 *   topk_idx, topk_w            as moe_route_topk (logits [T][E] fp32);
 *   expert_counts .. recv_src   as moe_dispatch_layout (capacity 0 = packed,
 *                               > 0 = padded [E][capacity]);
 *   recv_q + recv_scale         as moe_dispatch_fp8 (x [T][H] bf16 bits), or
 *   recv_x                      as moe_dispatch_bf16.
 * Extra constraints: H <= 2^20, T*H <= 2^40; bf16 needs H >= 64
 * (MOE_ERR_UNSUPPORTED otherwise).
 *
 * The kernel is a cooperative launch (every CTA resident) with two
 * grid-wide barriers kept in the workspace:
 *   workspace   device memory, 256-byte aligned, at least
 *               moe_route_dispatch_workspace_bytes(T, k, E, R) bytes (a
 *               value for the CURRENT device: it depends on its SM count).
 *               It carries state from call to call (a grid barrier, work
 *               counters, per-rank totals), so it must be ZERO before the
 *               first call and is then reserved for these two entry
 *               points; every call that completes leaves it ready for the
 *               next, whatever the sizes of either.  A wait inside the
 *               kernel gives up after 1 s and records MOE_ERR_TIMEOUT in
 *               *dev_status (the outputs are then incomplete); zero the
 *               workspace again before reusing it.  Calls that share a
 *               workspace must not overlap on the GPU.
 * Returns MOE_ERR_WORKSPACE for a missing, misaligned or short workspace,
 * MOE_ERR_CUDA if the device cannot run the cooperative launch.
 * T == 0 still launches (counts, offsets and recv_src are written).
 */
size_t moe_route_dispatch_workspace_bytes(int T, int k, int E, int R);
int moe_route_dispatch_fp8(const float *logits, int T, int E, int k, int renormalize, int R,
                           int capacity, const uint16_t *x, int H, int32_t *topk_idx,
                           float *topk_w, int32_t *expert_counts, int32_t *expert_src_counts,
                           int32_t *rank_counts, int32_t *expert_offsets, int32_t *dispatch_pos,
                           int32_t *recv_src, uint8_t *recv_q, float *recv_scale, int64_t rows,
                           void *workspace, size_t ws_bytes, int32_t *dev_status, void *stream);
int moe_route_dispatch_bf16(const float *logits, int T, int E, int k, int renormalize, int R,
                            int capacity, const uint16_t *x, int H, int32_t *topk_idx,
                            float *topk_w, int32_t *expert_counts, int32_t *expert_src_counts,
                            int32_t *rank_counts, int32_t *expert_offsets, int32_t *dispatch_pos,
                            int32_t *recv_src, uint16_t *recv_x, int64_t rows, void *workspace,
                            size_t ws_bytes, int32_t *dev_status, void *stream);

/*
 * moe_route_dispatch_ex_fp8 / moe_route_dispatch_ex_bf16 -- the same single
 * launch with the routing of moe_route_topk_ex (shared experts, replicas):
 * bit-identical to moe_route_topk_ex(..., tokens_per_rank = T / R), then
 * moe_dispatch_layout with k + n_shared slots and E_phys experts, then
 * moe_dispatch_fp8 (or _bf16).  logits stay [T][E] over the routed experts;
 * topk_idx / topk_w are [T][k + n_shared]; the layout outputs are sized by
 * E_phys (expert_counts [E_phys], expert_offsets [E_phys + 1],
 * expert_src_counts [E_phys][R]) and R must divide E_phys.  The table
 * arguments, their limits and their error behaviour are moe_route_topk_ex's;
 * a slot that gets -1 is left out of the layout (no row).  The workspace is
 * the one described above, at least moe_route_dispatch_workspace_bytes(T,
 * k + n_shared, E_phys, R) bytes, shared with the plain entry points.
 */
int moe_route_dispatch_ex_fp8(const float *logits, int T, int E, int k, int renormalize,
                              int n_shared, float shared_weight, const int32_t *replica_offsets,
                              const int32_t *replica_ids, int n_replica_ids, int E_phys, int R,
                              int capacity, const uint16_t *x, int H, int32_t *topk_idx,
                              float *topk_w, int32_t *expert_counts, int32_t *expert_src_counts,
                              int32_t *rank_counts, int32_t *expert_offsets, int32_t *dispatch_pos,
                              int32_t *recv_src, uint8_t *recv_q, float *recv_scale, int64_t rows,
                              void *workspace, size_t ws_bytes, int32_t *dev_status, void *stream);
int moe_route_dispatch_ex_bf16(const float *logits, int T, int E, int k, int renormalize,
                               int n_shared, float shared_weight, const int32_t *replica_offsets,
                               const int32_t *replica_ids, int n_replica_ids, int E_phys, int R,
                               int capacity, const uint16_t *x, int H, int32_t *topk_idx,
                               float *topk_w, int32_t *expert_counts, int32_t *expert_src_counts,
                               int32_t *rank_counts, int32_t *expert_offsets,
                               int32_t *dispatch_pos, int32_t *recv_src, uint16_t *recv_x,
                               int64_t rows, void *workspace, size_t ws_bytes, int32_t *dev_status,
                               void *stream);

/*
 * moe_combine_bf16 --gather each token's k expert outputs and form the
 * router-weighted sum.
 * Follows "Efficient and portable mixture-of-experts communication",
 * "Combinação" (the receiver reads the routing table for which row to read
 * and which weight to give it, and computes the weighted sum of the expert
 * contributions) and "Enabling trillion-parameter models on AWS EFA",
 * "Dağıtım/Birleştirme Gecikmesi" (bf16 combine; accumulation only at the
 * receiver).
 *
 *   out[g][h] = bf16_rne( acc ), acc = 0; for j = 0..k-1 ascending, slots
 *   with dispatch_pos == -1 skipped: acc = acc + (topk_w[g][j] *
 *   y[dispatch_pos[g][j]][h]), one binary32 multiply and one binary32 add
 *   per term (no fused multiply-add), so the result is bit-reproducible.
 *   y       [rows][H] bf16 bits (expert outputs, rows as laid out).
 *   topk_w  [T][k] fp32.
 *   out     [T][H] bf16 bits out.
 * T == 0 enqueues nothing.
 */
int moe_combine_bf16(const uint16_t *y, const int32_t *dispatch_pos,
                     const float *topk_w, int T, int H, int k, int64_t rows,
                     uint16_t *out, int32_t *dev_status, void *stream);

/*
 * moe_combine_bf16_long_form -- 1 when moe_combine_bf16 runs its long form
 * for these sizes (k <= 8, H % 16 == 0 and T*k*H*2 >= 2 GiB of rows read,
 * with y and out 32-byte aligned: 32-byte row loads, two rows at a time),
 * 0 otherwise or for invalid sizes.  Both forms give the same bits; this host
 * query only names the kernel that runs (for profiling and reports).
 */
int moe_combine_bf16_long_form(int T, int H, int k);

/*
 * moe_combine_fp8 -- moe_combine_bf16 with the expert rows in the dispatch's
 * FP8 format: E4M3 codes and one fp32 scale per 1x128 block (DeepSeek-V3
 * fragments: activations scaled per token per 128 channels), a payload of
 * H + H/32 bytes per row instead of 2H.
 *   out[g][h] = bf16_rne( acc ), acc = 0; for j = 0..k-1 ascending, slots
 *   with dispatch_pos == -1 skipped: acc = acc + (topk_w[g][j] *
 *   (decode(y_q[row][h]) * y_scale[row][h / 128])), each product and sum one
 *   binary32 operation (decode is exact), no fused multiply-add.
 *   y_q      [rows][H] E4M3 codes (16-byte aligned rows).
 *   y_scale  [rows][H/128] fp32, row-major.
 * H % 128 != 0 -> MOE_ERR_UNSUPPORTED.  T == 0 enqueues nothing.
 */
int moe_combine_fp8(const uint8_t *y_q, const float *y_scale, const int32_t *dispatch_pos,
                    const float *topk_w, int T, int H, int k, int64_t rows, uint16_t *out,
                    int32_t *dev_status, void *stream);

/*
 * Host-buffer entry points -- the path with the step's inputs and its result
 * in HOST memory.  The pages have no counterpart: these are deployment
 * variants of the entry points above, not steps of the method.  A serving
 * loop whose router logits and hidden states arrive from the host (a
 * CPU-side scheduler, a test harness, a process without a device allocator
 * of its own) hands host buffers to the library; each call enqueues, on
 * `stream` and in this order, the host -> device copies of the step's
 * inputs, the same kernels as the device-pointer entry points, and (for the
 * combine) the device -> host copy of the result.  Outputs are bit-identical
 * to those entry points.
 *
 * Every argument of the device-pointer entry point keeps its meaning, layout
 * and limits; the host buffers come in addition:
 *   logits_host [T][E] fp32, x_host [T][H] bf16 bits, out_host [T][H] bf16
 *   bits: host memory owned by the caller, read (written) by the copies.
 *   logits [T][E], x [T][H], out [T][H]: the DEVICE buffers the copies go
 *   through, owned by the caller, with the alignment rules above.
 *
 * Host memory.  With page-locked memory (cudaHostAlloc, cudaHostRegister,
 * torch's pin_memory) the copies are asynchronous: the call returns at once
 * and the copies overlap work on other streams.  The caller must then keep
 * logits_host / x_host unchanged, and leave out_host unread, until the
 * stream has passed the copies (an event or a stream synchronise).  Pageable
 * memory also works, but the runtime stages it and the call may block the
 * host thread until the copy has been staged (host -> device) or has
 * completed (device -> host); a stream being captured into a CUDA graph
 * accepts page-locked memory only (a capture error returns MOE_ERR_CUDA).
 *
 * Errors.  Every argument of every step is checked before anything is
 * enqueued (MOE_ERR_INVALID_ARG / _UNSUPPORTED / _WORKSPACE, as the
 * device-pointer entry points return them); a host pointer that is NULL
 * while T > 0 is MOE_ERR_INVALID_ARG.  A failed copy or launch returns
 * MOE_ERR_CUDA, and the steps before it may already be enqueued.  Kernel-
 * detected errors go to *dev_status as above.
 */

/*
 * moe_route_dispatch_fp8_host / moe_route_dispatch_bf16_host -- copy
 * logits_host into logits and x_host into x, then route, lay out and
 * dispatch.  flags = 0: the separate kernels, exactly moe_route_topk(logits,
 * ...), moe_dispatch_layout(...) with `workspace` of at least
 * moe_layout_workspace_bytes(T, k, E, R) bytes, and moe_dispatch_fp8 (or
 * _bf16).  flags = MOE_HOST_FUSED: the single cooperative launch of
 * moe_route_dispatch_fp8 (or _bf16), with that entry point's workspace rules
 * (zero-filled before first use, at least moe_route_dispatch_workspace_bytes(
 * T, k, E, R) bytes, not shared with the layout's).  Other flag bits are
 * MOE_ERR_INVALID_ARG.  The outputs are those of the entry points named.
 */
#define MOE_HOST_FUSED 1
int moe_route_dispatch_fp8_host(const float *logits_host, const uint16_t *x_host, int T, int E,
                                int k, int renormalize, int R, int capacity, int H, int flags,
                                float *logits, uint16_t *x, int32_t *topk_idx, float *topk_w,
                                int32_t *expert_counts, int32_t *expert_src_counts,
                                int32_t *rank_counts, int32_t *expert_offsets,
                                int32_t *dispatch_pos, int32_t *recv_src, uint8_t *recv_q,
                                float *recv_scale, int64_t rows, void *workspace, size_t ws_bytes,
                                int32_t *dev_status, void *stream);
int moe_route_dispatch_bf16_host(const float *logits_host, const uint16_t *x_host, int T, int E,
                                 int k, int renormalize, int R, int capacity, int H, int flags,
                                 float *logits, uint16_t *x, int32_t *topk_idx, float *topk_w,
                                 int32_t *expert_counts, int32_t *expert_src_counts,
                                 int32_t *rank_counts, int32_t *expert_offsets,
                                 int32_t *dispatch_pos, int32_t *recv_src, uint16_t *recv_x,
                                 int64_t rows, void *workspace, size_t ws_bytes,
                                 int32_t *dev_status, void *stream);

/*
 * moe_combine_bf16_host / moe_combine_fp8_host -- moe_combine_bf16 (or
 * _fp8) into the device buffer `out`, then a copy of out [T][H] into
 * out_host.  T == 0 enqueues nothing.
 */
int moe_combine_bf16_host(const uint16_t *y, const int32_t *dispatch_pos, const float *topk_w,
                          int T, int H, int k, int64_t rows, uint16_t *out, uint16_t *out_host,
                          int32_t *dev_status, void *stream);
int moe_combine_fp8_host(const uint8_t *y_q, const float *y_scale, const int32_t *dispatch_pos,
                         const float *topk_w, int T, int H, int k, int64_t rows, uint16_t *out,
                         uint16_t *out_host, int32_t *dev_status, void *stream);

/*
 * moe_quantize_e4m3 -- q[i] = e4m3(v[i]) with the converter moe_dispatch_fp8
 * uses (round to nearest even, saturating at +-448, NaN -> 0x7F).  Exposed
 * so the converter can be checked on every binary32 bit pattern.
 *   v  [n] fp32 (4-byte aligned);  q  [n] uint8 out.
 */
int moe_quantize_e4m3(const float *v, int64_t n, uint8_t *q, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_ROUTE_H */
