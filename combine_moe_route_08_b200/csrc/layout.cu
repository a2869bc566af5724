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
// order-free result); every position comes from prefix sums.
//
// Tokens are cut into chunks that never straddle two logical source ranks
// (at most 2048 slots each); one 1024-thread CTA owns a chunk and each of its
// 32 warps a contiguous run of at most 2 x 32 slots, which every lane keeps in
// registers (one load round trip per kernel).
//
//   k_layout_hist    chunk histogram (shared-memory atomics; small CTAs)
//                    -> workspace hist[chunk][E].
//   k_layout_assign  every CTA sums the histogram columns it needs (the base
//                    of its chunk inside each expert, the expert totals, its
//                    rank's source counts) with all its threads -- redundant
//                    but parallel, no serial tail -- scans the totals into
//                    offsets, builds per-warp histograms of its own slots,
//                    scans them over the warps, and ranks each slot among the
//                    equal experts of its warp step (equality mask + popc of
//                    the lower lanes) to get its row.  CTA 0 also writes
//                    counts, offsets and rank sums; the first chunk of each
//                    rank writes that rank's source-count column.
// The kernel boundary between the two is the only grid-wide ordering; nothing
// waits on another CTA.
//
// Small layouts (one chunk per logical rank and at most one slot per thread
// of an 8-CTA cluster: T*k <= 8192, e.g. the Mixtral-like workload) take a
// single launch instead: k_layout_cluster, one thread-block cluster of at
// most 8 CTAs.  Each CTA owns a run of whole ranks, counts them per warp, and
// publishes its per-expert totals in its own shared memory; one cluster
// barrier later every CTA reads the others' totals over distributed shared
// memory, scans, and ranks its slots exactly as k_layout_assign does.  The grid-wide ordering is then the hardware cluster
// barrier (all CTAs of a cluster are co-scheduled), not a kernel boundary
// plus a global round trip through the workspace.  Larger layouts keep the
// pair: with 4096 slots per SM (T = 4096, k = 8) the single cluster measured
// 11.9 against 9.0 us per layout, its per-warp equality masks and ranking
// steps then costing about 0.7 us each on eight SMs; at 1024 slots it saves
// about 0.9 us (5.1 against 5.9 us).
//
// The warp-level pieces (equality masks, per-warp histograms and bases, the
// block scan) are in layout_dev.cuh.
#include <algorithm>
#include <atomic>
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"
#include "layout_dev.cuh"

namespace moe {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
// 32-slot steps per warp.  2048-slot chunks: at prefill size (T = 32768,
// k = 8) 128 CTAs share the work instead of 32 with 8192-slot chunks, which
// measured 1079-1083 against 1086-1090 us per step; the decode workloads
// have one chunk per rank either way.
constexpr int kMaxSteps = 2;
constexpr int kChunkSlots = kThreads * kMaxSteps;  // 2048
// The placement kernel: kAssignThreads threads per chunk, each warp owning a
// run of at most kAssignSteps 32-slot steps.
constexpr int kAssignThreads = 1024;
constexpr int kAssignWarps = kAssignThreads / 32;
constexpr int kAssignSteps = kChunkSlots / kAssignThreads;
constexpr int kColBatch = 16;                      // 4-byte histogram loads in flight per thread
constexpr int kColBatch4 = 6;                      // 16-byte histogram loads in flight per thread

__device__ __forceinline__ void chunk_tokens(const LayoutGeom &G, int c, int &t0, int &t1)
{
    const int r = c / G.cpr;
    const int sub = c - r * G.cpr;
    const int rank_end = (r + 1) * G.Tr;
    t0 = min(r * G.Tr + sub * G.CT, rank_end);
    t1 = min(t0 + G.CT, rank_end);
}

// This warp's run of slots [w0, w1) inside chunk c, in 32-slot steps.
__device__ __forceinline__ void warp_run(const LayoutGeom &G, int c, int64_t &w0, int64_t &w1)
{
    int t0, t1;
    chunk_tokens(G, c, t0, t1);
    const int64_t i0 = static_cast<int64_t>(t0) * G.k, i1 = static_cast<int64_t>(t1) * G.k;
    const int64_t seg = static_cast<int64_t>(ceil_div(static_cast<int>(i1 - i0), kAssignWarps * 32)) * 32;
    const int w = threadIdx.x >> 5;
    w0 = min(i0 + w * seg, i1);
    w1 = min(w0 + seg, i1);
}

// The lane's slots of its warp run, loaded in one go (-1 past the end).
__device__ __forceinline__ void load_run(const int32_t *__restrict__ topk_idx, int64_t w0,
                                         int64_t w1, int (&e)[kAssignSteps])
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int s = 0; s < kAssignSteps; ++s) {
        const int64_t i = w0 + 32 * s + lane;
        e[s] = (i < w1) ? __ldg(topk_idx + i) : -1;
    }
}

// The histogram needs no order, so it runs in small CTAs: kHistThreads
// threads take the chunk's slots in strides, one shared-memory atomic per
// slot.  Small CTAs fit beside the route kernel's resident CTAs, so they are
// in place (waiting) when the route finishes, where a 1024-thread CTA must
// wait for a whole SM to drain first.
constexpr int kHistThreads = 256;
constexpr int kHistSlots = kChunkSlots / kHistThreads;  // slots per thread, at most

__global__ void __launch_bounds__(kHistThreads)
    k_layout_hist(const int32_t *__restrict__ topk_idx, LayoutGeom G,
                  int32_t *__restrict__ ws_hist, int32_t *__restrict__ dev_status)
{
    extern __shared__ int32_t h[];  // [E]
    const int E = G.E;
    const int c = blockIdx.x;
    int t0, t1;
    chunk_tokens(G, c, t0, t1);
    const int64_t i0 = static_cast<int64_t>(t0) * G.k, i1 = static_cast<int64_t>(t1) * G.k;
    for (int x = threadIdx.x; x < E; x += kHistThreads)
        h[x] = 0;
    pdl_trigger();  // the next kernel may take idle SM slots now; it waits for this one
    pdl_wait();
    int e[kHistSlots];
#pragma unroll
    for (int s = 0; s < kHistSlots; ++s) {
        const int64_t i = i0 + s * kHistThreads + threadIdx.x;
        e[s] = (i < i1) ? __ldg(topk_idx + i) : -1;
    }
    __syncthreads();
    bool bad = false;
#pragma unroll
    for (int s = 0; s < kHistSlots; ++s) {
        const bool valid = static_cast<unsigned>(e[s]) < static_cast<unsigned>(E);
        bad |= !valid && e[s] != -1;  // -1: an empty slot, or past the chunk's end
        if (valid)  // counts are order-free: one shared-memory atomic per slot
            atomicAdd(&h[e[s]], 1);
    }
    if (bad)
        report(dev_status, MOE_ERR_INVALID_ARG);
    __syncthreads();
    for (int x = threadIdx.x; x < E; x += kHistThreads)
        ws_hist[static_cast<size_t>(c) * E + x] = h[x];
}

// Histogram columns for chunk c of rank r (chunks [r0, r1) of that rank):
// slots of each expert in earlier chunks (before), in all chunks (total), in
// the rank's chunks (mine) and in chunks of earlier ranks (rstart).  P
// threads per column group each sum a contiguous share of the n chunk rows;
// V = 4 reads four experts per 16-byte load (E % 4 == 0, rows 16-byte
// aligned), V = 1 one per 4-byte load; B loads in flight per thread.  Share
// `part` writes rows 4*part .. 4*part+3 of out (before, total, mine, rstart).
template <int V, int B>
__device__ __forceinline__ void column_sums(const int32_t *__restrict__ ws_hist, int n, int c, int r0,
                                            int r1, int E, int P, int32_t *out)
{
    using Vec = typename std::conditional<V == 4, int4, int>::type;
    const int EV = E / V;
    const int xv = threadIdx.x % EV, part = threadIdx.x / EV;
    if (part >= P)
        return;
    const int per = ceil_div(n, P);
    const int cb = part * per, ce = min(n, cb + per);
    int before[V], total[V], mine[V], rstart[V];
#pragma unroll
    for (int q = 0; q < V; ++q)
        before[q] = total[q] = mine[q] = rstart[q] = 0;
    for (int c0 = cb; c0 < ce; c0 += B) {
        Vec v[B];
#pragma unroll
        for (int u = 0; u < B; ++u)
            v[u] = (c0 + u < ce)
                       ? __ldg(reinterpret_cast<const Vec *>(ws_hist + static_cast<size_t>(c0 + u) * E) +
                               xv)
                       : Vec{};
#pragma unroll
        for (int u = 0; u < B; ++u) {
            const int cc = c0 + u;
            const int *vv = reinterpret_cast<const int *>(&v[u]);
#pragma unroll
            for (int q = 0; q < V; ++q) {
                before[q] += (cc < c) ? vv[q] : 0;
                rstart[q] += (cc < r0) ? vv[q] : 0;
                total[q] += vv[q];
                mine[q] += (cc >= r0 && cc < r1) ? vv[q] : 0;
            }
        }
    }
#pragma unroll
    for (int q = 0; q < V; ++q) {
        const int x = V * xv + q;
        out[(4 * part) * E + x] = before[q];
        out[(4 * part + 1) * E + x] = total[q];
        out[(4 * part + 2) * E + x] = mine[q];
        out[(4 * part + 3) * E + x] = rstart[q];
    }
}

// Shares per histogram column: as many as the threads allow, at most
// kAssignWarps / 4 (kColBatch4 or kColBatch rows in flight per thread).
__host__ __device__ inline int column_shares(int E)
{
    const int per_share = (E % 4 == 0) ? E / 4 : E;
    const int p = kAssignThreads / per_share;
    return p < 1 ? 1 : (p > kAssignWarps / 4 ? kAssignWarps / 4 : p);
}

// Shared memory: wh[kAssignWarps][E] per-warp counts, then bases; parts[4P][E]
// column-sum shares; off[E + 1]; chb[E]; rbs[E]; tot[kAssignWarps + 1].
__global__ void __launch_bounds__(kAssignThreads)
    k_layout_assign(const int32_t *__restrict__ topk_idx, LayoutGeom G, int capacity, int64_t rows,
                    const int32_t *__restrict__ ws_hist, int32_t *__restrict__ expert_counts,
                    int32_t *__restrict__ expert_src_counts, int32_t *__restrict__ rank_counts,
                    int32_t *__restrict__ expert_offsets, int32_t *__restrict__ dispatch_pos,
                    int32_t *__restrict__ recv_src, int32_t *__restrict__ private_pos,
                    int32_t *__restrict__ dev_status)
{
    extern __shared__ int32_t sm[];
    const int E = G.E, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int nb = key_bits(E);
    const int P = column_shares(E);
    int32_t *wh = sm;                   // [kAssignWarps][E] per-warp counts, then bases
    int32_t *parts = wh + kAssignWarps * E;   // [4P][E] column-sum shares
    int32_t *off = parts + 4 * P * E;   // [E + 1] expert totals, then their scan
    int32_t *chb = off + E + 1;         // [E] slots of e in earlier chunks
    int32_t *rbs = chb + E;             // [E] slots of e in chunks of earlier ranks
    int32_t *tot = rbs + E;             // [kAssignWarps + 1]
    const int c = blockIdx.x;

    int64_t w0, w1;
    warp_run(G, c, w0, w1);
    for (int x = threadIdx.x; x < kAssignWarps * E; x += kAssignThreads)
        wh[x] = 0;  // before the wait: nothing upstream is read
    pdl_trigger();  // the next kernel may take idle SM slots now; it waits for this one
    pdl_wait();
    int e[kAssignSteps];
    load_run(topk_idx, w0, w1, e);  // in flight while the columns are summed

    // histogram columns: base of this chunk inside each expert (earlier
    // chunks), expert totals, and this chunk's rank column of the
    // per-source-rank counts.  P threads per expert each sum a contiguous
    // part of the chunks (coalesced over experts); the parts meet below.
    const int n = G.nchunks;
    const int r = c / G.cpr;
    if (E % 4 == 0)  // CTA-uniform
        column_sums<4, kColBatch4>(ws_hist, n, c, r * G.cpr, (r + 1) * G.cpr, E, P, parts);
    else
        column_sums<1, kColBatch>(ws_hist, n, c, r * G.cpr, (r + 1) * G.cpr, E, P, parts);
    __syncthreads();  // wh zeroed by every thread before any warp counts into it
    // per-warp counts of this CTA's slots (order-free: shared-memory atomics)
    warp_count(e, w0, w1, E, wh + w * E);
    for (int x = threadIdx.x; x < E; x += kAssignThreads) {
        int before = 0, total = 0, mine = 0, rstart = 0;
        for (int part = 0; part < P; ++part) {
            before += parts[(4 * part) * E + x];
            total += parts[(4 * part + 1) * E + x];
            mine += parts[(4 * part + 2) * E + x];
            rstart += parts[(4 * part + 3) * E + x];
        }
        off[x] = total;
        chb[x] = before;
        rbs[x] = rstart;
        if (c == 0)
            expert_counts[x] = total;
        if (c == r * G.cpr)  // first chunk of its rank writes the rank's column
            expert_src_counts[static_cast<size_t>(x) * G.R + r] = mine;
    }
    __syncthreads();
    block_exclusive_scan<kAssignWarps>(off, E, tot);  // off[e] = slots of experts < e; off[E] = total
    if (c == 0) {
        for (int x = threadIdx.x; x <= E; x += kAssignThreads)
            expert_offsets[x] = (capacity == 0) ? off[x] : x * capacity;
        const int L = E / G.R;
        for (int rr = threadIdx.x; rr < G.R; rr += kAssignThreads)
            rank_counts[rr] = off[(rr + 1) * L] - off[rr * L];
    }
    // per-warp base of each expert's positions: earlier chunks + earlier warps
    warp_bases_par<kAssignWarps>(wh, chb, E);
    __syncthreads();
    int32_t *mywh = wh + w * E;

    // rank every slot among equal experts, in slot order
    bool dropped = false, bad_row = false;
#pragma unroll
    for (int s = 0; s < kAssignSteps; ++s) {
        if (w0 + 32 * s >= w1)
            break;
        const int64_t i = w0 + 32 * s + lane;
        const bool valid = static_cast<unsigned>(e[s]) < static_cast<unsigned>(E);
        const int p = rank_step(e[s], E, nb, mywh);
        if (i < w1) {
            int64_t row = -1, prow = -1;
            bool hole = false;  // private mode: packed row left empty by a dropped slot
            if (valid) {
                if (capacity == 0)
                    row = off[e[s]] + p;
                else if (p < capacity)
                    row = static_cast<int64_t>(e[s]) * capacity + p;
                else
                    dropped = true;
                if (G.max_m > 0 && row >= 0) {
                    // position among this rank's slots of the expert
                    const int pr = p - rbs[e[s]];
                    if (pr < G.max_m) {
                        prow = (static_cast<int64_t>(e[s]) * G.R + r) * G.max_m + pr;
                    } else {
                        dropped = true;
                        hole = true;
                    }
                }
            }
            if (row >= rows) {  // cannot happen for a consistent layout; never write past rows
                bad_row = true;
                row = -1;
            }
            dispatch_pos[i] = hole ? -1 : static_cast<int32_t>(row);
            if (row >= 0)
                recv_src[row] = hole ? -1 : static_cast<int32_t>(i);
            if (G.max_m > 0)
                private_pos[i] = static_cast<int32_t>(prow);
        }
    }
    if (dropped)
        report(dev_status, MOE_ERR_CAPACITY);
    if (bad_row)
        report(dev_status, MOE_ERR_INVALID_ARG);

    // rows that no slot fills -> -1
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kAssignThreads;
    const int64_t first = static_cast<int64_t>(c) * kAssignThreads + threadIdx.x;
    if (capacity == 0) {
        for (int64_t r = off[E] + first; r < rows; r += stride)
            recv_src[r] = -1;
    } else {
        for (int x = c; x < E; x += gridDim.x) {
            const int filled = min(off[x + 1] - off[x], capacity);
            for (int p = filled + threadIdx.x; p < capacity; p += kAssignThreads)
                recv_src[static_cast<int64_t>(x) * capacity + p] = -1;
        }
        for (int64_t r = static_cast<int64_t>(E) * capacity + first; r < rows; r += stride)
            recv_src[r] = -1;
    }
}

// ---------------------------------------------------------------------------
// Single-launch layout for small layouts (one chunk per rank): one cluster.

constexpr int kClusterMax = 8;        // CTAs of the cluster (portable cluster size)
constexpr int kClusterSteps = 2;      // 32-slot steps per warp, at most
constexpr int kClusterMaxE = 1024;

__device__ __forceinline__ unsigned cluster_ctarank()
{
    unsigned r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// p (this CTA's shared memory) as seen in CTA `rank` of the cluster, loaded.
__device__ __forceinline__ int32_t ld_peer_smem(const int32_t *p, unsigned rank)
{
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
    uint32_t ra;
    int32_t v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
    asm volatile("ld.shared::cluster.b32 %0, [%1];" : "=r"(v) : "r"(ra) : "memory");
    return v;
}

// CTA b of the cluster owns chunks (= ranks) [b*cpb, b*cpb + cpb); warp w
// serves chunk b*cpb + w / wpc, the (w % wpc)-th run of seg slots of it.
// Shared memory: wh[32][E] per-warp counts, then in-CTA bases; tot[E] this
// CTA's totals (read by the other CTAs); off[E+1] totals over the cluster,
// then their exclusive scan; bef[E] slots of each expert in earlier CTAs;
// cst[cpb][E] in-CTA base at each chunk's first warp (private mode);
// scan scratch [33].
__global__ void __launch_bounds__(kThreads)
    k_layout_cluster(const int32_t *__restrict__ topk_idx, LayoutGeom G, int cpb, int wpc, int seg,
                     int capacity, int64_t rows, int32_t *__restrict__ expert_counts,
                     int32_t *__restrict__ expert_src_counts, int32_t *__restrict__ rank_counts,
                     int32_t *__restrict__ expert_offsets, int32_t *__restrict__ dispatch_pos,
                     int32_t *__restrict__ recv_src, int32_t *__restrict__ private_pos,
                     int32_t *__restrict__ dev_status)
{
    extern __shared__ int32_t sm[];
    const int E = G.E, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int nb = key_bits(E);
    int32_t *wh = sm;
    int32_t *tot = wh + kWarps * E;
    int32_t *off = tot + E;
    int32_t *bef = off + E + 1;
    int32_t *cst = bef + E;
    int32_t *scr = cst + cpb * E;
    const unsigned b = cluster_ctarank();
    const unsigned C = gridDim.x;

    // this warp's run [w0, w1) of the slots of chunk c (empty for spare warps)
    const int lc = w / wpc;
    const int c = static_cast<int>(b) * cpb + lc;
    const bool has_chunk = lc < cpb && c < G.nchunks;
    int64_t w0 = 0, w1 = 0;
    if (has_chunk) {
        const int64_t i0 = static_cast<int64_t>(c) * G.Tr * G.k;
        const int64_t i1 = i0 + static_cast<int64_t>(G.Tr) * G.k;
        w0 = min(i0 + static_cast<int64_t>(w % wpc) * seg, i1);
        w1 = min(w0 + seg, i1);
    }
    for (int x = threadIdx.x; x < kWarps * E; x += kThreads)
        wh[x] = 0;
    pdl_trigger();  // the next kernel may take idle SM slots now; it waits for this one
    pdl_wait();
    int e[kClusterSteps];
    bool bad = false;
#pragma unroll
    for (int s = 0; s < kClusterSteps; ++s) {
        const int64_t i = w0 + 32 * s + lane;
        e[s] = (i < w1) ? __ldg(topk_idx + i) : -1;
        bad |= (i < w1) && e[s] != -1 && static_cast<unsigned>(e[s]) >= static_cast<unsigned>(E);
    }
    if (bad)
        report(dev_status, MOE_ERR_INVALID_ARG);
    __syncthreads();
    warp_count(e, w0, w1, E, wh + w * E);
    __syncthreads();

    // per expert: in-CTA exclusive prefix over the warps (slot order), each
    // chunk's count (its rank's source-count column) and the CTA total
    for (int x = threadIdx.x; x < E; x += kThreads) {
        int run = 0;
        for (int q = 0; q < cpb; ++q) {
            const int start = run;
            if (G.max_m > 0)
                cst[q * E + x] = start;
            for (int ww = q * wpc; ww < (q + 1) * wpc; ++ww) {
                const int t = wh[ww * E + x];
                wh[ww * E + x] = run;
                run += t;
            }
            const int cq = static_cast<int>(b) * cpb + q;
            if (cq < G.nchunks)
                expert_src_counts[static_cast<size_t>(x) * G.R + cq] = run - start;
        }
        tot[x] = run;
    }
    cluster_arrive();  // publishes tot (release) ...
    cluster_wait();    // ... and sees every CTA's (acquire)
    for (int x = threadIdx.x; x < E; x += kThreads) {
        int before = 0, total = 0;
        for (unsigned bb = 0; bb < C; ++bb) {
            const int v = ld_peer_smem(tot + x, bb);
            total += v;
            before += (bb < b) ? v : 0;
        }
        off[x] = total;
        bef[x] = before;
        if (b == 0)
            expert_counts[x] = total;
    }
    cluster_arrive();  // done reading the other CTAs' tot; waited for before exit
    __syncthreads();
    block_exclusive_scan<kWarps>(off, E, scr);  // off[e] = slots of experts < e; off[E] = total
    if (b == 0) {
        for (int x = threadIdx.x; x <= E; x += kThreads)
            expert_offsets[x] = (capacity == 0) ? off[x] : x * capacity;
        const int L = E / G.R;
        for (int rr = threadIdx.x; rr < G.R; rr += kThreads)
            rank_counts[rr] = off[(rr + 1) * L] - off[rr * L];
    }

    // rank every slot among equal experts, in slot order
    int32_t *mywh = wh + w * E;
    bool dropped = false, bad_row = false;
#pragma unroll
    for (int s = 0; s < kClusterSteps; ++s) {
        if (w0 + 32 * s >= w1)
            break;  // warp-uniform
        const int64_t i = w0 + 32 * s + lane;
        const bool valid = static_cast<unsigned>(e[s]) < static_cast<unsigned>(E);
        const int p = rank_step(e[s], E, nb, mywh);  // in-CTA position among equal experts
        if (i < w1) {
            int64_t row = -1, prow = -1;
            bool hole = false;  // private mode: packed row left empty by a dropped slot
            if (valid) {
                const int pe = bef[e[s]] + p;  // position inside the expert
                if (capacity == 0)
                    row = off[e[s]] + pe;
                else if (pe < capacity)
                    row = static_cast<int64_t>(e[s]) * capacity + pe;
                else
                    dropped = true;
                if (G.max_m > 0 && row >= 0) {
                    const int pr = p - cst[lc * E + e[s]];  // among this rank's slots of e
                    if (pr < G.max_m) {
                        prow = (static_cast<int64_t>(e[s]) * G.R + c) * G.max_m + pr;
                    } else {
                        dropped = true;
                        hole = true;
                    }
                }
            }
            if (row >= rows) {  // cannot happen for a consistent layout; never write past rows
                bad_row = true;
                row = -1;
            }
            dispatch_pos[i] = hole ? -1 : static_cast<int32_t>(row);
            if (row >= 0)
                recv_src[row] = hole ? -1 : static_cast<int32_t>(i);
            if (G.max_m > 0)
                private_pos[i] = static_cast<int32_t>(prow);
        }
    }
    if (dropped)
        report(dev_status, MOE_ERR_CAPACITY);
    if (bad_row)
        report(dev_status, MOE_ERR_INVALID_ARG);

    // rows that no slot fills -> -1
    const int64_t stride = static_cast<int64_t>(C) * kThreads;
    const int64_t first = static_cast<int64_t>(b) * kThreads + threadIdx.x;
    if (capacity == 0) {
        for (int64_t r = off[E] + first; r < rows; r += stride)
            recv_src[r] = -1;
    } else {
        for (int x = static_cast<int>(b); x < E; x += static_cast<int>(C)) {
            const int filled = min(off[x + 1] - off[x], capacity);
            for (int p = filled + threadIdx.x; p < capacity; p += kThreads)
                recv_src[static_cast<int64_t>(x) * capacity + p] = -1;
        }
        for (int64_t r = static_cast<int64_t>(E) * capacity + first; r < rows; r += stride)
            recv_src[r] = -1;
    }
    cluster_wait();  // no CTA exits while another may still read its tot
}

size_t assign_smem_bytes(int E)
{
    return (static_cast<size_t>(kAssignWarps + 4 * column_shares(E) + 3) * E + 1 + kAssignWarps + 1) *
           sizeof(int32_t);
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
    g.CT = std::max(1, kChunkSlots / k);  // at most 2048 slots per chunk
    g.cpr = std::max(1, ceil_div(g.Tr, g.CT));
    g.nchunks = R * g.cpr;
    g.max_m = 0;
    return g;
}

size_t layout_workspace_bytes(const LayoutGeom &g)
{
    const size_t hist = static_cast<size_t>(g.nchunks) * g.E * sizeof(int32_t);
    return std::max<size_t>(256, (hist + 255) / 256 * 256);
}

namespace {

// The single-launch plan for a geometry, or ok = false when it does not pay
// or fit: more than one chunk per rank, more slots than one per thread of
// the CTAs, E beyond the kernel's limit, shared memory beyond the device's
// opt-in limit, or a device that cannot schedule such a cluster.
struct ClusterPlan {
    bool ok = false;
    int C = 0, cpb = 0, wpc = 0, seg = 0;
    size_t smem = 0;
};

size_t cluster_smem_bytes(int E, int cpb)
{
    return (static_cast<size_t>(kWarps + 3 + cpb) * E + 1 + kWarps + 1) * sizeof(int32_t);
}

// Whether this device can run one cluster of kClusterMax CTAs of kThreads
// threads with `smem` bytes each (queried once per device for the largest
// shared-memory size the plan allows).
bool cluster_schedulable(size_t smem)
{
    constexpr int kMaxDev = 64;
    static std::atomic<int> state[kMaxDev];  // 0 unknown, 1 yes, 2 no
    static std::atomic<int> optin[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
        cudaGetLastError();
        return false;
    }
    int st = state[dev].load(std::memory_order_acquire);
    if (st == 0) {
        int limit = 0;
        bool ok = cudaDeviceGetAttribute(&limit, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess;
        const size_t probe = std::min<size_t>(static_cast<size_t>(limit), cluster_smem_bytes(kClusterMaxE, 8));
        ok = ok && cudaFuncSetAttribute(k_layout_cluster, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(probe)) == cudaSuccess;
        int n = 0;
        if (ok) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(kClusterMax);
            cfg.blockDim = dim3(kThreads);
            cfg.dynamicSmemBytes = probe;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = kClusterMax;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            ok = cudaOccupancyMaxActiveClusters(&n, k_layout_cluster, &cfg) == cudaSuccess && n >= 1;
        }
        if (!ok)
            cudaGetLastError();
        optin[dev].store(ok ? static_cast<int>(probe) : 0, std::memory_order_relaxed);
        st = ok ? 1 : 2;
        state[dev].store(st, std::memory_order_release);
    }
    return st == 1 && smem <= static_cast<size_t>(optin[dev].load(std::memory_order_relaxed));
}

ClusterPlan cluster_plan(const LayoutGeom &g)
{
    ClusterPlan p;
    if (g.cpr != 1 || g.E > kClusterMaxE)
        return p;
    const int n = g.nchunks;  // one chunk per rank
    int C = std::min(kClusterMax, n);
    const int cpb = ceil_div(n, C);
    if (cpb > kWarps)
        return p;
    const int wpc = kWarps / cpb;
    const int slots = g.Tr * g.k;
    if (static_cast<int64_t>(cpb) * slots > kThreads)
        return p;  // more work per SM than the two-kernel form spreads over more SMs
    const int seg = round_up(ceil_div(slots, wpc), 32);
    if (seg > 32 * kClusterSteps)
        return p;
    C = ceil_div(n, cpb);
    const size_t smem = cluster_smem_bytes(g.E, cpb);
    if (!cluster_schedulable(smem))
        return p;
    p.ok = true;
    p.C = C;
    p.cpb = cpb;
    p.wpc = wpc;
    p.seg = seg;
    p.smem = smem;
    return p;
}

}  // namespace

int layout_launches(const LayoutGeom &g) { return cluster_plan(g).ok ? 1 : 2; }

cudaError_t dispatch_layout(const int32_t *topk_idx, const LayoutGeom &g, int capacity, int64_t rows,
                            int32_t *expert_counts, int32_t *expert_src_counts,
                            int32_t *rank_counts, int32_t *expert_offsets, int32_t *dispatch_pos,
                            int32_t *recv_src, int32_t *private_pos, void *workspace,
                            int32_t *dev_status, cudaStream_t s)
{
    const ClusterPlan cp = cluster_plan(g);
    if (cp.ok) {
        cudaError_t err = cudaFuncSetAttribute(k_layout_cluster, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(cp.smem));
        if (err != cudaSuccess)
            return err;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(cp.C);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = cp.smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = cp.C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        return cudaLaunchKernelEx(&cfg, k_layout_cluster, topk_idx, g, cp.cpb, cp.wpc, cp.seg,
                                  capacity, rows, expert_counts, expert_src_counts, rank_counts,
                                  expert_offsets, dispatch_pos, recv_src, private_pos, dev_status);
    }
    int32_t *hist = static_cast<int32_t *>(workspace);
    cudaError_t err = launch_pdl(k_layout_hist, dim3(g.nchunks), dim3(kHistThreads),
                                 g.E * sizeof(int32_t), s, topk_idx, g, hist, dev_status);
    if (err != cudaSuccess)
        return err;
    const size_t smem = assign_smem_bytes(g.E);
    if (smem > 48 * 1024) {
        err = cudaFuncSetAttribute(k_layout_assign, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   static_cast<int>(smem));
        if (err != cudaSuccess)
            return err;
    }
    return launch_pdl(k_layout_assign, dim3(g.nchunks), dim3(kAssignThreads), smem, s, topk_idx, g, capacity,
                      rows, hist, expert_counts, expert_src_counts, rank_counts, expert_offsets,
                      dispatch_pos, recv_src, private_pos, dev_status);
}

}  // namespace moe
