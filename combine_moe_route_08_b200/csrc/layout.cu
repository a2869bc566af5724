// layout.cu -- per-expert counts, offsets and index maps (deterministic).
//
// "Enabling trillion-parameter models on AWS EFA", "Dağıtım ve Birleştirme":
// dispatch counts the tokens of each expert by atomic accumulation in shared
// memory, then keeps summing the counts cumulatively to find the offsets that
// pack tokens into contiguous per-expert buffers; "Gönderme ve Alma
// Arabellekleri": counts first, then every sender knows where its writes go.
// "Efficient and portable mixture-of-experts communication", "Despacho": one
// routing warp counts, and the source indices are kept so that combine knows
// where each row came from.
//
// The pages' receiver fills its buffers in a nondeterministic order; here the
// slots of an expert take consecutive rows in ascending slot index g*k + j, so
// the layout is bit-reproducible.  Atomics only ever build histograms (an
// order-free result); every position comes from prefix sums:
//
//   k_layout_count  (one CTA per chunk of tokens inside one logical rank)
//       shared-memory histogram of the chunk (warp-aggregated with
//       __match_any_sync), stored to the workspace; the last CTA to finish
//       (atomic ticket, no waiting) turns the chunk histograms into per-chunk
//       exclusive prefixes per expert, the per-(expert, source rank) counts,
//       the expert totals, their exclusive scan (offsets) and rank totals.
//   k_layout_assign (one CTA per chunk again)
//       each warp owns a contiguous run of the chunk's slots; per-warp
//       histograms -> exclusive prefix over the warps -> in-warp rank of each
//       slot among equal experts (__match_any_sync + popc of the lower lanes)
//       gives the slot's row; recv_src is the inverse map, -1 elsewhere.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kLayoutThreads = 256;
constexpr int kLayoutWarps = kLayoutThreads / 32;
constexpr size_t kTicketBytes = 256;

__device__ __forceinline__ void chunk_tokens(const LayoutGeom &G, int c, int &t0, int &t1)
{
    const int r = c / G.cpr;
    const int sub = c - r * G.cpr;
    const int rank_end = (r + 1) * G.Tr;
    t0 = min(r * G.Tr + sub * G.CT, rank_end);
    t1 = min(t0 + G.CT, rank_end);
}

__device__ __forceinline__ unsigned lanemask_lt()
{
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// In-place exclusive scan of a[0..n) by 256 threads (n <= 1024); a[n] gets
// the total.  `tot` is 9 ints of scratch shared memory.
__device__ void block_exclusive_scan(int32_t *a, int n, int32_t *tot)
{
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int per = ceil_div(n, kLayoutThreads);  // <= 4
    const int b = tid * per;
    int loc[4];
    int sum = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        loc[u] = (u < per && b + u < n) ? a[b + u] : 0;
        sum += loc[u];
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(kFullMask, incl, off);
        if (lane >= off)
            incl += t;
    }
    if (lane == 31)
        tot[wid] = incl;
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int w = 0; w < kLayoutWarps; ++w) {
            const int t = tot[w];
            tot[w] = run;
            run += t;
        }
        tot[kLayoutWarps] = run;
    }
    __syncthreads();
    int run = tot[wid] + incl - sum;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        if (u < per && b + u < n) {
            a[b + u] = run;
            run += loc[u];
        }
    }
    if (tid == 0)
        a[n] = tot[kLayoutWarps];
    __syncthreads();
}

__global__ void __launch_bounds__(kLayoutThreads)
    k_layout_count(const int32_t *__restrict__ topk_idx, LayoutGeom G, int capacity,
                   int32_t *__restrict__ ws_hist, unsigned *__restrict__ ws_ticket,
                   int32_t *__restrict__ expert_counts, int32_t *__restrict__ expert_src_counts,
                   int32_t *__restrict__ rank_counts, int32_t *__restrict__ expert_offsets,
                   int32_t *__restrict__ dev_status)
{
    extern __shared__ int32_t sm[];  // [E + 1] histogram, later the scan
    __shared__ int32_t scan_tot[kLayoutWarps + 1];
    __shared__ bool is_last;
    const int E = G.E;
    const int tid = threadIdx.x, lane = tid & 31;
    const int c = blockIdx.x;

    for (int e = tid; e <= E; e += kLayoutThreads)
        sm[e] = 0;
    __syncthreads();

    int t0, t1;
    chunk_tokens(G, c, t0, t1);
    const int64_t i0 = static_cast<int64_t>(t0) * G.k, i1 = static_cast<int64_t>(t1) * G.k;
    bool bad = false;
    for (int64_t base = i0; base < i1; base += kLayoutThreads) {  // CTA-uniform trips
        const int64_t i = base + tid;
        const int e = (i < i1) ? __ldg(topk_idx + i) : -1;
        const bool valid = static_cast<unsigned>(e) < static_cast<unsigned>(E);
        bad |= (i < i1) && !valid && e != -1;
        const unsigned mask = __match_any_sync(kFullMask, valid ? e : (0x40000000 | lane));
        if (valid && lane == __ffs(mask) - 1)
            atomicAdd(&sm[e], __popc(mask));
    }
    if (bad)
        report(dev_status, MOE_ERR_INVALID_ARG);
    __syncthreads();

    int32_t *mine = ws_hist + static_cast<size_t>(c) * E;
    for (int e = tid; e < E; e += kLayoutThreads)
        mine[e] = sm[e];
    __threadfence();
    __syncthreads();
    if (tid == 0)
        is_last = (atomicAdd(ws_ticket, 1u) == gridDim.x - 1);
    __syncthreads();
    if (!is_last)
        return;
    __threadfence();

    // ---- last CTA: per expert, walk the chunks in order ----
    const int n = G.nchunks;
    for (int e = tid; e < E; e += kLayoutThreads) {
        int run = 0, src = 0;
        for (int c0 = 0; c0 < n; c0 += 8) {
            int v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                v[u] = (c0 + u < n) ? __ldcg(ws_hist + static_cast<size_t>(c0 + u) * E + e) : 0;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int cc = c0 + u;
                if (cc < n) {
                    ws_hist[static_cast<size_t>(cc) * E + e] = run;  // chunk's base in e
                    run += v[u];
                    src += v[u];
                    if (cc % G.cpr == G.cpr - 1) {
                        expert_src_counts[static_cast<size_t>(e) * G.R + cc / G.cpr] = src;
                        src = 0;
                    }
                }
            }
        }
        expert_counts[e] = run;
        sm[e] = run;
    }
    __syncthreads();
    block_exclusive_scan(sm, E, scan_tot);  // sm[e] = slots of experts < e, sm[E] = total
    for (int e = tid; e <= E; e += kLayoutThreads)
        expert_offsets[e] = (capacity == 0) ? sm[e] : e * capacity;
    const int L = E / G.R;
    for (int r = tid; r < G.R; r += kLayoutThreads)
        rank_counts[r] = sm[(r + 1) * L] - sm[r * L];
    if (tid == 0)
        *ws_ticket = 0u;  // leave the workspace reusable
}

__global__ void __launch_bounds__(kLayoutThreads)
    k_layout_assign(const int32_t *__restrict__ topk_idx, LayoutGeom G, int capacity, int64_t rows,
                    const int32_t *__restrict__ ws_hist, const int32_t *__restrict__ expert_counts,
                    const int32_t *__restrict__ expert_offsets, int32_t *__restrict__ dispatch_pos,
                    int32_t *__restrict__ recv_src, int32_t *__restrict__ dev_status)
{
    extern __shared__ int32_t sm[];
    const int E = G.E;
    int32_t *wh = sm;                      // [8][E] per-warp running base
    int32_t *ob = sm + kLayoutWarps * E;   // [E + 1] expert row base
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int c = blockIdx.x;

    for (int x = tid; x < kLayoutWarps * E; x += kLayoutThreads)
        wh[x] = 0;
    for (int e = tid; e <= E; e += kLayoutThreads)
        ob[e] = expert_offsets[e];
    __syncthreads();

    int t0, t1;
    chunk_tokens(G, c, t0, t1);
    const int64_t i0 = static_cast<int64_t>(t0) * G.k, i1 = static_cast<int64_t>(t1) * G.k;
    const int64_t seg = static_cast<int64_t>(ceil_div(static_cast<int>(i1 - i0), kLayoutWarps * 32)) * 32;
    const int64_t w0 = min(i0 + w * seg, i1), w1 = min(w0 + seg, i1);
    int32_t *mywh = wh + w * E;

    // pass A: per-warp histogram of its run of slots
    for (int64_t base = w0; base < w1; base += 32) {  // warp-uniform trips
        const int64_t i = base + lane;
        const int e = (i < w1) ? __ldg(topk_idx + i) : -1;
        const bool valid = static_cast<unsigned>(e) < static_cast<unsigned>(E);
        const unsigned mask = __match_any_sync(kFullMask, valid ? e : (0x40000000 | lane));
        if (valid && lane == __ffs(mask) - 1)
            mywh[e] += __popc(mask);
        __syncwarp();
    }
    __syncthreads();

    // pass B: base of each warp = chunk base in e + slots of e in earlier warps
    for (int e = tid; e < E; e += kLayoutThreads) {
        int run = ws_hist[static_cast<size_t>(c) * E + e];
#pragma unroll
        for (int ww = 0; ww < kLayoutWarps; ++ww) {
            const int t = wh[ww * E + e];
            wh[ww * E + e] = run;
            run += t;
        }
    }
    __syncthreads();

    // pass C: rank inside the warp among equal experts -> row
    bool dropped = false;
    for (int64_t base = w0; base < w1; base += 32) {
        const int64_t i = base + lane;
        const int e = (i < w1) ? __ldg(topk_idx + i) : -1;
        const bool valid = static_cast<unsigned>(e) < static_cast<unsigned>(E);
        const unsigned mask = __match_any_sync(kFullMask, valid ? e : (0x40000000 | lane));
        const int p = valid ? mywh[e] + __popc(mask & lanemask_lt()) : 0;
        __syncwarp();
        if (valid && lane == __ffs(mask) - 1)
            mywh[e] += __popc(mask);
        __syncwarp();
        if (i < w1) {
            int row = -1;
            if (valid) {
                if (capacity == 0)
                    row = ob[e] + p;
                else if (p < capacity)
                    row = e * capacity + p;
                else
                    dropped = true;
            }
            if (row >= rows) {  // cannot happen for a consistent layout; never write past rows
                report(dev_status, MOE_ERR_INVALID_ARG);
                row = -1;
            }
            dispatch_pos[i] = row;
            if (row >= 0)
                recv_src[row] = static_cast<int32_t>(i);
        }
    }
    if (dropped)
        report(dev_status, MOE_ERR_CAPACITY);

    // rows that no slot fills -> -1
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kLayoutThreads;
    if (capacity == 0) {
        for (int64_t r = ob[E] + static_cast<int64_t>(c) * kLayoutThreads + tid; r < rows; r += stride)
            recv_src[r] = -1;
    } else {
        for (int e = c; e < E; e += gridDim.x) {
            const int filled = min(expert_counts[e], capacity);
            for (int p = filled + tid; p < capacity; p += kLayoutThreads)
                recv_src[static_cast<int64_t>(e) * capacity + p] = -1;
        }
        for (int64_t r = static_cast<int64_t>(E) * capacity + static_cast<int64_t>(c) * kLayoutThreads + tid;
             r < rows; r += stride)
            recv_src[r] = -1;
    }
}

}  // namespace

LayoutGeom layout_geom(int T, int k, int E, int R)
{
    LayoutGeom g;
    g.T = T;
    g.k = k;
    g.E = E;
    g.R = R;
    g.Tr = T / R;
    g.CT = std::max(1, 2048 / k);  // about 2048 slots per chunk
    g.cpr = std::max(1, ceil_div(g.Tr, g.CT));
    g.nchunks = R * g.cpr;
    return g;
}

size_t layout_workspace_bytes(const LayoutGeom &g)
{
    const size_t hist = static_cast<size_t>(g.nchunks) * g.E * sizeof(int32_t);
    return kTicketBytes + (hist + 255) / 256 * 256;
}

cudaError_t dispatch_layout(const int32_t *topk_idx, const LayoutGeom &g, int capacity, int64_t rows,
                            int32_t *expert_counts, int32_t *expert_src_counts,
                            int32_t *rank_counts, int32_t *expert_offsets, int32_t *dispatch_pos,
                            int32_t *recv_src, void *workspace, int32_t *dev_status,
                            cudaStream_t s)
{
    unsigned *ticket = static_cast<unsigned *>(workspace);
    int32_t *hist = reinterpret_cast<int32_t *>(static_cast<char *>(workspace) + kTicketBytes);
    const size_t smem1 = (g.E + 1) * sizeof(int32_t);
    k_layout_count<<<g.nchunks, kLayoutThreads, smem1, s>>>(topk_idx, g, capacity, hist, ticket,
                                                            expert_counts, expert_src_counts,
                                                            rank_counts, expert_offsets, dev_status);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess)
        return err;
    const size_t smem2 = (static_cast<size_t>(kLayoutWarps) * g.E + g.E + 1) * sizeof(int32_t);
    k_layout_assign<<<g.nchunks, kLayoutThreads, smem2, s>>>(topk_idx, g, capacity, rows, hist,
                                                             expert_counts, expert_offsets,
                                                             dispatch_pos, recv_src, dev_status);
    return cudaGetLastError();
}

}  // namespace moe
