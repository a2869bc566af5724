// route_dispatch.cu -- router, layout and dispatch in one persistent
// cooperative kernel.
//
// "Enabling trillion-parameter models on AWS EFA", "Dağıtım ve Birleştirme":
// the dispatch kernel itself counts the tokens of each expert (atomic
// accumulation in shared memory within a block), sums the counts into
// offsets, and packs the tokens into contiguous per-expert buffers at those
// offsets; "Gönderme ve Alma Arabellekleri": the counts go first, then every
// sender knows where its writes land.  "Efficient and portable
// mixture-of-experts communication", "Despacho": a routing warp counts while
// the other warps move the tokens.  The three steps that the separate entry
// points run as five launches (route, two layout kernels, dispatch) run here
// as one launch with one grid-wide barrier.
//
// Phases (tokens are cut into chunks inside one logical source rank, about
// one chunk per resident CTA):
//   A  route: one warp per token (route_warp, the same code as the route
//      kernel); the chunk's slots are counted per expert in shared memory;
//      the count row goes to hist[chunk] and is added (global atomics) to the
//      per-rank totals rt[rank].
//   -- grid barrier: every count is in --
//   C  place: every CTA sums rt into the expert totals and offsets; for each
//      of its chunks it forms the chunk's base inside every expert (earlier
//      ranks from rt, earlier chunks of its rank from hist), ranks the
//      chunk's slots among equal experts (the layout kernel's warp-level
//      counting), writes dispatch_pos / recv_src, and publishes the chunk as
//      placed (a flag set to this launch's epoch).
//   D  pack: the x rows are cut into tickets of up to 960 16-byte units
//      (FP8: 16 channels each; a 128-channel block never straddles two
//      tickets).  One warp per CTA takes tickets from a grid-wide counter,
//      one ahead, waits until the chunks the next ticket touches are placed
//      and copies its tokens' rows into shared memory; the 15 other warps
//      pack the current ticket, two units per thread with all their x loads
//      in flight: read x, quantise (FP8), store to the k rows.  Tickets
//      spread the bandwidth-bound packing over the SMs as they drain, which
//      a static split by chunk does not (measured: CTAs finished up to 2x
//      apart).
// Results are bit-identical to moe_route_topk + moe_dispatch_layout +
// moe_dispatch_fp8 / _bf16.
//
// State kept in the workspace between launches, all of which a zeroed
// workspace starts consistent with and every completed launch leaves so:
//   - the barrier word (arrival count | generation): the count returns to 0;
//   - rt, in a region of fixed place and size (R * E <= 2^20), nothing else
//     writes: the last CTA to finish placing zeroes the part it used;
//   - the "placed" flags: tagged with this launch's epoch (generation + 1,
//     top bit set), so stale flags of other launches, and the non-negative
//     counts that a differently sized launch left in that memory, never
//     match.
// Every wait (the barrier, a chunk flag) gives up after 1 s (%globaltimer)
// and records MOE_ERR_TIMEOUT; the launch is cooperative, so the driver
// guarantees that every CTA is resident.
#include <algorithm>
#include <type_traits>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "dispatch_dev.cuh"
#include "kernels.cuh"
#include "layout_dev.cuh"
#include "route_dev.cuh"

namespace moe {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kPackers = kThreads - 32;            // threads that pack (warps 1..15)
constexpr int kUnitsPerThread = 2;                 // 16-byte units a packer holds per ticket
constexpr int kTicketUnits = kPackers * kUnitsPerThread;
constexpr int kPosCap = 2048;                      // rows of one ticket's tokens in shared memory

// Units per pack ticket: kTicketUnits, or fewer when the tokens a ticket can
// touch (at most TU / upt + 2) would need more than kPosCap rows; a multiple
// of 8 so that a 128-channel FP8 block (8 units) never straddles two tickets.
__host__ __device__ inline int ticket_units(int upt, int k)
{
    const int max_tok = kPosCap / k - 2;
    const int64_t tu = static_cast<int64_t>(max_tok) * upt;
    const int t = static_cast<int>(tu < kTicketUnits ? tu : kTicketUnits);
    return t >= 8 ? t / 8 * 8 : t;
}

// Shared memory (int32 units): phase A's counts [E], phase C's per-warp rows
// and scans (kWarps * E + 2E + 1 + kWarps + 1), then the pack phase's two
// ticket row buffers, kept apart so that packing can start while the last
// flag of C is still being published.
__host__ __device__ inline int kPosOffset(int E)
{
    return (kWarps * E + 2 * E + 1 + kWarps + 1 + 31) / 32 * 32;
}
constexpr int kSumBatch = 12;                      // 4-byte table loads in flight per thread
constexpr int kSumBatch4 = 4;                      // 16-byte table loads in flight per thread

constexpr int kMaxSteps = 8;                       // 32-slot steps per warp
constexpr int kChunkSlots = kThreads * kMaxSteps;  // 4096 slots per chunk at most
constexpr int kHeadInts = 64;                      // barrier word, ticket and done counters
constexpr size_t kRtInts = size_t(1) << 20;        // rt region: R * E <= 1024 * 1024
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

struct FusedGeom {
    int T, k, E, R;
    int Tr;       // tokens per logical source rank
    int CT;       // tokens per chunk
    int cpr;      // chunks per rank
    int nchunks;  // R * cpr
    int G;        // CTAs
};

struct FusedArgs {
    const float *logits;
    int El;  // routed experts (logits per token)
    int kr;  // routed slots per token; slots kr .. k-1 are the shared experts
    int renormalize;
    // shared experts and replicas (as moe_route_topk_ex); ex_on = 0: the
    // chosen logical experts are the layout's experts
    int ex_on;
    float shared_weight;
    const int32_t *replica_offsets;  // [El + n_shared + 1] or nullptr
    const int32_t *replica_ids;
    int n_replica_ids;
    const uint4 *x;
    int H;
    int capacity;
    int64_t rows;
    int32_t *topk_idx;
    float *topk_w;
    int32_t *expert_counts;
    int32_t *expert_src_counts;
    int32_t *rank_counts;
    int32_t *expert_offsets;
    int32_t *dispatch_pos;
    int32_t *recv_src;
    void *recv;         // u8 codes [rows][H] or bf16 [rows][H]
    float *recv_scale;  // [rows][H/128] (FP8)
    int32_t *ws;
    int32_t *dev_status;
};

// Workspace layout in int32 units.
struct WsLayout {
    size_t flags, rt, hist, total;
};

__host__ __device__ inline WsLayout ws_layout(const FusedGeom &g)
{
    auto up = [](size_t n) { return (n + kHeadInts - 1) / kHeadInts * kHeadInts; };
    WsLayout L;
    L.rt = kHeadInts;                                          // [R][E], fixed region
    L.flags = L.rt + kRtInts;                                  // [nchunks]
    L.hist = L.flags + up(static_cast<size_t>(g.nchunks));      // [nchunks][E]
    L.total = L.hist + up(static_cast<size_t>(g.nchunks) * g.E);
    return L;
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long *p)
{
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(unsigned *p, unsigned v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned long long globaltimer()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Grid-wide barrier on one 64-bit word: low half = arrivals, high half =
// generation.  The last CTA to arrive turns (gen, G) into (gen + 1, 0) with
// one atomic; the others wait for the generation to move past gen0 (the
// value every CTA read at launch start).  Returns false, with MOE_ERR_TIMEOUT
// recorded, if that takes more than the limit.  Every thread calls it.
__device__ bool grid_barrier(unsigned long long *word, unsigned gen0, int32_t *dev_status)
{
    __shared__ int ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned long long old = atomicAdd(word, 1ull);
        int good = 1;
        if (static_cast<unsigned>(old) == gridDim.x - 1) {
            atomicAdd(word, (1ull << 32) - gridDim.x);
        } else {
            const unsigned long long t0 = globaltimer();
            while (static_cast<unsigned>(ld_acquire_u64(word) >> 32) == gen0) {
                if (globaltimer() - t0 > kWaitLimitNs) {
                    good = 0;
                    report(dev_status, MOE_ERR_TIMEOUT);
                    break;
                }
                __nanosleep(20);
            }
        }
        __threadfence();
        ok = good;
    }
    __syncthreads();
    return ok != 0;
}

__device__ __forceinline__ void chunk_tokens(const FusedGeom &G, int c, int &t0, int &t1)
{
    const int r = c / G.cpr;
    const int sub = c - r * G.cpr;
    const int rank_end = (r + 1) * G.Tr;
    t0 = min(r * G.Tr + sub * G.CT, rank_end);
    t1 = min(t0 + G.CT, rank_end);
}

__device__ __forceinline__ int chunk_of(const FusedGeom &G, int g)
{
    const int r = g / G.Tr;
    return r * G.cpr + (g - r * G.Tr) / G.CT;
}

// Wait until chunk c is placed in this launch; false after the time limit.
__device__ __forceinline__ bool wait_placed(const unsigned *flags, int c, unsigned epoch,
                                            int32_t *dev_status)
{
    if (ld_acquire(flags + c) == epoch)
        return true;
    const unsigned long long t0 = globaltimer();
    while (ld_acquire(flags + c) != epoch) {
        if (globaltimer() - t0 > kWaitLimitNs) {
            report(dev_status, MOE_ERR_TIMEOUT);
            return false;
        }
        __nanosleep(64);
    }
    return true;
}

// out[part * E + x] = sum of rows [r0, r1) of a [rows][E] int32 table at
// column x, rows split into P contiguous shares (out holds P * E ints); loads
// kSumBatch at a time, all in flight.  Every thread calls it; ends with
// __syncthreads().  Used for a CTA's later chunks (only when chunks outnumber
// CTAs); a second inlined copy of the 16-byte form below pushed the kernel
// past its 64-register budget (spills), so that form serves the first chunk
// only.
__device__ void sum_rows(const int32_t *tab, int E, int r0, int r1, int P, int32_t *out)
{
    for (int idx = threadIdx.x; idx < P * E; idx += kThreads) {
        const int x = idx % E, part = idx / E;
        const int n = max(0, r1 - r0);
        const int per = (n + P - 1) / P;
        const int b = r0 + part * per, e = min(r1, b + per);
        int acc = 0;
        for (int rr = b; rr < e; rr += kSumBatch) {
            int v[kSumBatch];
#pragma unroll
            for (int u = 0; u < kSumBatch; ++u)
                v[u] = (rr + u < e) ? __ldcg(tab + static_cast<size_t>(rr + u) * E + x) : 0;
#pragma unroll
            for (int u = 0; u < kSumBatch; ++u)
                acc += v[u];
        }
        out[part * E + x] = acc;
    }
    __syncthreads();
}

// Column sums of the int32 tables for placing a chunk, in one pass of loads:
// rows [0, R) of rt (each adds to the expert total; those of ranks < rb also
// to the chunk's base) and rows [h0, h1) of hist (base only).  The
// R + (h1 - h0) rows are split into Q contiguous shares per column, Q <= Qmax
// as large as the CTA's threads allow.  V = 4: a thread reads four columns
// per 16-byte load (needs E % 4 == 0; rows are then 16-byte aligned); V = 1:
// one column per 4-byte load.  Each thread keeps B loads in flight.  Writes
// tot_out / bef_out [Q][E] and returns Q.  Every thread calls it; ends with
// __syncthreads().
template <int V, int B>
__device__ int sum_totals_and_base(const int32_t *rt, int R, int rb, const int32_t *hist, int h0,
                                   int h1, int E, int Qmax, int32_t *tot_out, int32_t *bef_out)
{
    using Vec = typename std::conditional<V == 4, int4, int>::type;
    const int n = R + (h1 - h0);
    const int EV = E / V;
    const int Q = max(1, min(min(kThreads / EV, Qmax), n));
    const int per = (n + Q - 1) / Q;
    for (int idx = threadIdx.x; idx < Q * EV; idx += kThreads) {
        const int xv = idx % EV, part = idx / EV;
        const int b = part * per, e = min(n, b + per);
        int total[V], before[V];
#pragma unroll
        for (int q = 0; q < V; ++q)
            total[q] = before[q] = 0;
        for (int j0 = b; j0 < e; j0 += B) {
            Vec val[B];
#pragma unroll
            for (int u = 0; u < B; ++u) {
                const int j = j0 + u;
                const int32_t *row = (j < R) ? rt + static_cast<size_t>(j) * E
                                             : hist + static_cast<size_t>(h0 + j - R) * E;
                val[u] = (j < e) ? __ldcg(reinterpret_cast<const Vec *>(row) + xv) : Vec{};
            }
#pragma unroll
            for (int u = 0; u < B; ++u) {  // rows past e hold zeros
                const int j = j0 + u;
                const int *vv = reinterpret_cast<const int *>(&val[u]);
#pragma unroll
                for (int q = 0; q < V; ++q) {
                    total[q] += (j < R) ? vv[q] : 0;
                    before[q] += (j < rb || j >= R) ? vv[q] : 0;
                }
            }
        }
#pragma unroll
        for (int q = 0; q < V; ++q) {
            tot_out[part * E + V * xv + q] = total[q];
            bef_out[part * E + V * xv + q] = before[q];
        }
    }
    __syncthreads();
    return Q;
}

__device__ __forceinline__ int sum_totals_and_base(const int32_t *rt, int R, int rb,
                                                   const int32_t *hist, int h0, int h1, int E,
                                                   int Qmax, int32_t *tot_out, int32_t *bef_out)
{
    if (E % 4 == 0)  // CTA-uniform
        return sum_totals_and_base<4, kSumBatch4>(rt, R, rb, hist, h0, h1, E, Qmax, tot_out,
                                                  bef_out);
    return sum_totals_and_base<1, kSumBatch>(rt, R, rb, hist, h0, h1, E, Qmax, tot_out, bef_out);
}

template <int NPL, bool FP8>
__global__ void __launch_bounds__(kThreads, (NPL <= 12) ? 2 : 1)
    k_route_dispatch(FusedArgs A, FusedGeom G)
{
    extern __shared__ int32_t sm[];
    __shared__ unsigned s_gen0;
    __shared__ int s_last;
    __shared__ int s_tick[2];
    const int E = G.E, k = G.k, R = G.R;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const WsLayout L = ws_layout(G);
    unsigned long long *bar = reinterpret_cast<unsigned long long *>(A.ws);
    unsigned *ticket = reinterpret_cast<unsigned *>(A.ws + 2);
    unsigned *done = reinterpret_cast<unsigned *>(A.ws + 3);
    int32_t *rt = A.ws + L.rt;
    unsigned *flags = reinterpret_cast<unsigned *>(A.ws + L.flags);
    int32_t *hist = A.ws + L.hist;

    if (tid == 0)
        s_gen0 = static_cast<unsigned>(ld_acquire_u64(bar) >> 32);
    __syncthreads();
    const unsigned gen0 = s_gen0, epoch = (gen0 + 1u) | 0x80000000u;

    // ---- A: route this CTA's chunks and count their slots per expert
    if (blockIdx.x == 0 && tid == 0)
        *ticket = 0;  // used only after the barrier
    for (int c = blockIdx.x; c < G.nchunks; c += gridDim.x) {
        int32_t *h = sm;  // [E]
        for (int x = tid; x < E; x += kThreads)
            h[x] = 0;
        __syncthreads();
        int t0, t1;
        chunk_tokens(G, c, t0, t1);
        const int src_r = c / G.cpr;  // a chunk's tokens share one source rank
        for (int g = t0 + w; g < t1; g += kWarps) {  // warp-uniform
            int my_e;
            float my_w;
            if (A.ex_on)  // uniform; two call sites keep the plain form's registers
                route_warp<NPL>(A.logits + static_cast<size_t>(g) * A.El, A.El, A.kr,
                                A.renormalize, my_e, my_w);
            else
                route_warp<NPL>(A.logits + static_cast<size_t>(g) * E, E, k, A.renormalize,
                                my_e, my_w);
            if (lane < k) {
                int phys = my_e;
                float wt = my_w;
                if (A.ex_on) {
                    // shared experts El .. El + k - kr - 1 after the routed ones;
                    // every logical expert mapped to the replica of the token's rank
                    const int l = (lane < A.kr) ? my_e : A.El + (lane - A.kr);
                    wt = (lane < A.kr) ? my_w : A.shared_weight;
                    phys = l;
                    if (A.replica_offsets != nullptr) {
                        const int a = A.replica_offsets[l], b = A.replica_offsets[l + 1];
                        if (a < 0 || b <= a || b > A.n_replica_ids)
                            phys = -1;
                        else
                            phys = A.replica_ids[a + src_r % (b - a)];
                    }
                    if (phys < 0 || phys >= E) {
                        report(A.dev_status, MOE_ERR_INVALID_ARG);
                        phys = -1;
                    }
                }
                A.topk_idx[static_cast<size_t>(g) * k + lane] = phys;
                A.topk_w[static_cast<size_t>(g) * k + lane] = wt;
                if (phys >= 0)
                    atomicAdd(&h[phys], 1);
            }
        }
        __syncthreads();
        int32_t *rtr = rt + static_cast<size_t>(c / G.cpr) * E;
        for (int x = tid; x < E; x += kThreads) {
            const int v = h[x];
            hist[static_cast<size_t>(c) * E + x] = v;
            if (v != 0)
                atomicAdd(rtr + x, v);
        }
        __syncthreads();
    }
    if (!grid_barrier(bar, gen0, A.dev_status))
        return;

    // ---- C: offsets, then place each of this CTA's chunks
    int32_t *wh = sm;                   // [kWarps][E] per-warp counts, then bases
    int32_t *off = wh + kWarps * E;     // [E + 1] expert totals, then their scan
    int32_t *chb = off + E + 1;         // [E] base of the chunk inside each expert
    int32_t *tot = chb + E;             // [kWarps + 1]
    const int nb = key_bits(E);

    // The first pack ticket is requested now; its answer is needed only when
    // packing starts.
    unsigned first_ticket = 0;
    if (tid == 0)
        first_ticket = atomicAdd(ticket, 1u);

    // The slots of the first chunk, then one pass of loads for the expert
    // totals and that chunk's base inside each expert (P threads per expert,
    // the shares meeting in the per-warp rows, not yet in use).
    const int c_first = blockIdx.x;  // this CTA's first chunk (none if >= nchunks)
    const int r_first = (c_first < G.nchunks) ? c_first / G.cpr : 0;
    const int h0_first = (c_first < G.nchunks) ? r_first * G.cpr : 0;
    const int h1_first = (c_first < G.nchunks) ? c_first : 0;
    int e_first[kMaxSteps];
    {
        int t0, t1;
        chunk_tokens(G, min(c_first, G.nchunks - 1), t0, t1);
        const int64_t i0 = static_cast<int64_t>(t0) * k, i1 = static_cast<int64_t>(t1) * k;
        const int64_t seg =
            static_cast<int64_t>(ceil_div(static_cast<int>(i1 - i0), kWarps * 32)) * 32;
        const int64_t w0 = min(i0 + w * seg, i1), w1 = min(w0 + seg, i1);
#pragma unroll
        for (int s = 0; s < kMaxSteps; ++s) {
            const int64_t i = w0 + 32 * s + lane;
            e_first[s] = (c_first < G.nchunks && i < w1) ? __ldcg(A.topk_idx + i) : -1;
        }
    }
    constexpr int kQ = kWarps / 2;  // shares per column: totals in wh rows [0, kQ), bases after
    const int Q1 = sum_totals_and_base(rt, R, r_first, hist, h0_first, h1_first, E, kQ, wh,
                                       wh + kQ * E);
    for (int x = tid; x < E; x += kThreads) {
        int total = 0, before = 0;
        for (int part = 0; part < Q1; ++part) {
            total += wh[part * E + x];
            before += wh[(kQ + part) * E + x];
        }
        off[x] = total;
        chb[x] = before;
    }
    __syncthreads();
    if (blockIdx.x == 0)
        for (int x = tid; x < E; x += kThreads)
            A.expert_counts[x] = off[x];
    block_exclusive_scan<kWarps>(off, E, tot);  // off[e] = slots of experts < e
    if (blockIdx.x == 0) {
        for (int x = tid; x <= E; x += kThreads)
            A.expert_offsets[x] = (A.capacity == 0) ? off[x] : x * A.capacity;
        const int Lr = E / R;
        for (int r = tid; r < R; r += kThreads)
            A.rank_counts[r] = off[(r + 1) * Lr] - off[r * Lr];
    }
    // rows that no slot fills -> -1
    {
        const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
        const int64_t first = static_cast<int64_t>(blockIdx.x) * kThreads + tid;
        if (A.capacity == 0) {
            for (int64_t r = off[E] + first; r < A.rows; r += stride)
                A.recv_src[r] = -1;
        } else {
            for (int x = blockIdx.x; x < E; x += gridDim.x) {
                const int filled = min(off[x + 1] - off[x], A.capacity);
                for (int p = filled + tid; p < A.capacity; p += kThreads)
                    A.recv_src[static_cast<int64_t>(x) * A.capacity + p] = -1;
            }
            for (int64_t r = static_cast<int64_t>(E) * A.capacity + first; r < A.rows; r += stride)
                A.recv_src[r] = -1;
        }
    }

    bool dropped = false, bad_row = false;
    for (int c = blockIdx.x; c < G.nchunks; c += gridDim.x) {
        const int r = c / G.cpr;
        int t0, t1;
        chunk_tokens(G, c, t0, t1);
        const int64_t i0 = static_cast<int64_t>(t0) * k, i1 = static_cast<int64_t>(t1) * k;
        const int64_t seg =
            static_cast<int64_t>(ceil_div(static_cast<int>(i1 - i0), kWarps * 32)) * 32;
        const int64_t w0 = min(i0 + w * seg, i1), w1 = min(w0 + seg, i1);
        int e[kMaxSteps];
        const int cfirst = r * G.cpr;
        if (c == c_first) {
#pragma unroll
            for (int s = 0; s < kMaxSteps; ++s)
                e[s] = e_first[s];
        } else {
#pragma unroll
            for (int s = 0; s < kMaxSteps; ++s) {
                const int64_t i = w0 + 32 * s + lane;
                e[s] = (i < w1) ? __ldcg(A.topk_idx + i) : -1;
            }
            // base of the chunk inside each expert: slots of earlier ranks
            // (rank rows 0..r-1), then of the earlier chunks of its rank
            const int P = max(1, min(kThreads / E, kWarps / 2));
            sum_rows(rt, E, 0, r, P, wh);
            sum_rows(hist, E, cfirst, c, P, wh + P * E);
            for (int x = tid; x < E; x += kThreads) {
                int before = 0;
                for (int part = 0; part < 2 * P; ++part)
                    before += wh[part * E + x];
                chb[x] = before;
            }
        }
        if (c == cfirst)  // the rank's first chunk writes its source-count column
            for (int x = tid; x < E; x += kThreads)
                A.expert_src_counts[static_cast<size_t>(x) * R + r] =
                    __ldcg(rt + static_cast<size_t>(r) * E + x);
        __syncthreads();
        for (int x = tid; x < kWarps * E; x += kThreads)
            wh[x] = 0;
        __syncthreads();
        int32_t *mywh = wh + w * E;
        warp_histogram(e, w0, w1, E, nb, mywh);
        __syncthreads();
        warp_bases_par<kWarps>(wh, chb, E);
        __syncthreads();
#pragma unroll
        for (int s = 0; s < kMaxSteps; ++s) {
            if (w0 + 32 * s >= w1)
                break;  // warp-uniform
            const int64_t i = w0 + 32 * s + lane;
            const bool valid = static_cast<unsigned>(e[s]) < static_cast<unsigned>(E);
            const int p = rank_step(e[s], E, nb, mywh);
            if (i < w1) {
                int64_t row = -1;
                if (valid) {
                    if (A.capacity == 0)
                        row = off[e[s]] + p;
                    else if (p < A.capacity)
                        row = static_cast<int64_t>(e[s]) * A.capacity + p;
                    else
                        dropped = true;
                }
                if (row >= A.rows) {  // cannot happen for validated sizes; never write past rows
                    bad_row = true;
                    row = -1;
                }
                A.dispatch_pos[i] = static_cast<int32_t>(row);
                if (row >= 0)
                    A.recv_src[row] = static_cast<int32_t>(i);
            }
        }
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            st_release(flags + c, epoch);
        }
    }
    if (dropped)
        report(A.dev_status, MOE_ERR_CAPACITY);
    if (bad_row)
        report(A.dev_status, MOE_ERR_INVALID_ARG);
    // this CTA has read rt for the last time; the last CTA to get here
    // returns it to zero at the end of the kernel (the count's answer is
    // only needed then)
    __syncthreads();
    unsigned done_before = 0;
    if (tid == 0)  // the reads of rt have all returned: no fence is needed
        done_before = atomicAdd(done, 1u);

    // ---- D: pack tickets of TU 16-byte units taken from the grid-wide
    // counter.  Warp 0 takes ticket n + 1, waits until every chunk it touches
    // is placed and copies its tokens' rows into shared memory while warps
    // 1..15 pack ticket n, each thread holding up to kUnitsPerThread units
    // with all their x loads in flight at once.
    const int H = A.H;
    const int upt = FP8 ? H / 16 : H / 8;  // 16-byte units per token
    const int TU = ticket_units(upt, k);
    const int64_t units = static_cast<int64_t>(G.T) * upt;
    const int64_t ntick = (units + TU - 1) / TU;
    int32_t *spos = sm + kPosOffset(E);  // [2][kPosCap], apart from C's arrays
    bool ok = true;  // warp 0: every wait ended in time
    auto take = [&](int slot, bool first) {  // warp 0 only
        int t = 0;
        if (lane == 0)
            t = static_cast<int>(first ? first_ticket : atomicAdd(ticket, 1u));
        t = __shfl_sync(kFullMask, t, 0);
        if (t < ntick && ok) {
            const int64_t u0 = static_cast<int64_t>(t) * TU;
            const int64_t u1 = min(u0 + TU, units);
            // The ticket's units are contiguous in x (32 bytes each for FP8,
            // 16 for bf16): one bulk L2 prefetch of them, issued before the
            // waits, so the packers' loads of ticket n + 1 find x in L2.  In
            // 10-step graphs, same outputs: dsv3 155.4 -> 152.0 us, prefill
            // 1098.0 -> 1091.8, kimi unchanged (224.4 / 224.9).
            if (lane == 0) {
                constexpr int ub = FP8 ? 32 : 16;
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(
                                 reinterpret_cast<const uint8_t *>(A.x) + u0 * ub),
                             "r"(static_cast<uint32_t>((u1 - u0) * ub))
                             : "memory");
            }
            const int ga = static_cast<int>(u0 / upt), gb = static_cast<int>((u1 - 1) / upt);
            const int ca = chunk_of(G, ga), cb = chunk_of(G, gb);
            for (int c = ca + lane; c <= cb; c += 32)
                if (!wait_placed(flags, c, epoch, A.dev_status))
                    ok = false;
            ok = __all_sync(kFullMask, ok);
            const int n = (gb - ga + 1) * k;  // <= kPosCap by the choice of TU
            for (int i = lane; ok && i < n; i += 32)
                spos[slot * kPosCap + i] = __ldcg(A.dispatch_pos + static_cast<size_t>(ga) * k + i);
        }
        if (lane == 0)
            s_tick[slot] = ok ? t : INT32_MAX;  // a failed wait ends the CTA's packing
    };
    if (w == 0)
        take(0, true);
    __syncthreads();
    int cur = 0;
    for (;;) {
        const int t = s_tick[cur];
        if (t >= ntick)
            break;  // CTA-uniform
        if (w == 0) {
            take(cur ^ 1, false);
        } else {
            const int64_t u0 = static_cast<int64_t>(t) * TU;
            const int64_t u1 = min(u0 + TU, units);
            const int ga = static_cast<int>(u0 / upt);
            const int32_t *rows_t = spos + cur * kPosCap;
            int g[kUnitsPerThread], v[kUnitsPerThread];
            bool act[kUnitsPerThread];
#pragma unroll
            for (int i = 0; i < kUnitsPerThread; ++i) {
                const int64_t u = u0 + (tid - 32) + i * kPackers;
                act[i] = u < u1;
                g[i] = act[i] ? static_cast<int>(u / upt) : 0;
                v[i] = act[i] ? static_cast<int>(u - static_cast<int64_t>(g[i]) * upt) : 0;
            }
            if (FP8) {
                uint4 xa[kUnitsPerThread], xb[kUnitsPerThread];
#pragma unroll
                for (int i = 0; i < kUnitsPerThread; ++i) {
                    xa[i] = make_uint4(0, 0, 0, 0);
                    xb[i] = make_uint4(0, 0, 0, 0);
                    if (act[i]) {
                        const uint4 *xr = A.x + static_cast<size_t>(g[i]) * (H / 8);
                        xa[i] = ld_stream_v4(xr + 2 * v[i]);
                        xb[i] = ld_stream_v4(xr + 2 * v[i] + 1);
                    }
                }
                uint8_t *recv_q = static_cast<uint8_t *>(A.recv);
                const int S = H / 128;
#pragma unroll
                for (int i = 0; i < kUnitsPerThread; ++i) {
                    float sc;
                    const uint4 q = quant_e4m3_x16(xa[i], xb[i], sc);  // all lanes (shuffles)
                    if (!act[i])
                        continue;
                    const int32_t *rr = rows_t + (g[i] - ga) * k;
                    for (int j = 0; j < k; ++j) {
                        const int r = rr[j];
                        if (r < 0)
                            continue;
                        st_stream_v4(recv_q + static_cast<size_t>(r) * H + 16 * v[i], q);
                        if ((v[i] & 7) == 0)
                            __stcs(A.recv_scale + static_cast<size_t>(r) * S + (v[i] >> 3), sc);
                    }
                }
            } else {
                uint4 d[kUnitsPerThread];
#pragma unroll
                for (int i = 0; i < kUnitsPerThread; ++i)
                    d[i] = act[i] ? ld_stream_v4(A.x + static_cast<size_t>(g[i]) * upt + v[i])
                                  : make_uint4(0, 0, 0, 0);
                uint4 *recv_x = static_cast<uint4 *>(A.recv);
#pragma unroll
                for (int i = 0; i < kUnitsPerThread; ++i) {
                    if (!act[i])
                        continue;
                    const int32_t *rr = rows_t + (g[i] - ga) * k;
                    for (int j = 0; j < k; ++j) {
                        const int r = rr[j];
                        if (r >= 0)
                            st_stream_v4(recv_x + static_cast<size_t>(r) * upt + v[i], d[i]);
                    }
                }
            }
        }
        __syncthreads();
        cur ^= 1;
    }
    if (tid == 0)
        s_last = (done_before == gridDim.x - 1) ? 1 : 0;
    __syncthreads();
    if (s_last) {  // every CTA has read rt: return it to zero for the next launch
        for (int i = tid; i < R * E; i += kThreads)
            rt[i] = 0;
        if (tid == 0)
            *done = 0;
    }
    pdl_trigger();
}

size_t smem_bytes(const FusedGeom &g)
{
    return (static_cast<size_t>(kPosOffset(g.E)) + 2 * kPosCap) * sizeof(int32_t);
}

using KernelFn = void (*)(FusedArgs, FusedGeom);

template <bool FP8>
KernelFn pick(int E)
{
    const int need = ceil_div(E, 32);
    if (need <= 1) return k_route_dispatch<1, FP8>;
    if (need <= 2) return k_route_dispatch<2, FP8>;
    if (need <= 4) return k_route_dispatch<4, FP8>;
    if (need <= 8) return k_route_dispatch<8, FP8>;
    if (need <= 12) return k_route_dispatch<12, FP8>;
    if (need <= 16) return k_route_dispatch<16, FP8>;
    if (need <= 24) return k_route_dispatch<24, FP8>;
    return k_route_dispatch<32, FP8>;
}

// Chunk geometry for a grid of at most gmax resident CTAs: about gmax / R
// chunks per rank (at least one), each at most kChunkSlots slots.  The grid:
// enough CTAs for every chunk and every pack ticket, at most gmax.
FusedGeom make_geom(int T, int k, int E, int R, int gmax, int64_t units)
{
    FusedGeom g;
    g.T = T;
    g.k = k;
    g.E = E;
    g.R = R;
    g.Tr = T / R;
    const int want = std::max(1, gmax / R);
    g.CT = std::max(1, std::min(ceil_div(std::max(g.Tr, 1), want), kChunkSlots / k));
    g.cpr = std::max(1, ceil_div(g.Tr, g.CT));
    g.nchunks = R * g.cpr;
    const int64_t ntick = (units + kTicketUnits - 1) / kTicketUnits;  // at least
    g.G = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(gmax, std::max<int64_t>(g.nchunks, ntick))));
    return g;
}

// Resident CTAs of the kernel on the current device (0 on error).  The
// answer is remembered per (device, kernel, shared memory): the occupancy
// query is not free and the answer never changes.
struct ResidentKey {
    int dev;
    KernelFn fn;
    size_t smem;
    int value;
};

int query_resident(KernelFn fn, size_t smem);

int max_resident(KernelFn fn, size_t smem)
{
    static std::mutex mu;
    static std::vector<ResidentKey> known;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (const ResidentKey &r : known)
            if (r.dev == dev && r.fn == fn && r.smem == smem)
                return r.value;
    }
    const int v = query_resident(fn, smem);
    if (v > 0) {
        std::lock_guard<std::mutex> lock(mu);
        known.push_back(ResidentKey{dev, fn, smem, v});
    }
    return v;
}

int query_resident(KernelFn fn, size_t smem)
{
    int dev = 0, nsm = 0, per = 0, coop = 0, optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess || !coop ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return 0;
    // The limit is a property of the kernel, shared by every geometry: it is
    // raised to the most the device allows next to the kernel's static
    // shared memory (never lowered to one geometry's need, which would break
    // a larger geometry whose answer is already cached).
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess)
        return 0;
    const size_t limit = static_cast<size_t>(optin) - fa.sharedSizeBytes;
    if (smem > limit)
        return 0;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(limit)) != cudaSuccess)
        return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, fn, kThreads, smem) != cudaSuccess)
        return 0;
    return nsm * per;
}

// Geometry on the current device, the grid sized from the kernel's occupancy.
// k and E are the layout's slots per token and experts; El, the logits per
// token, picks the kernel (logits per lane).
bool device_geom(int T, int k, int E, int R, int H, bool fp8, int El, FusedGeom &g, KernelFn &fn)
{
    fn = fp8 ? pick<true>(El) : pick<false>(El);
    FusedGeom probe;
    probe.E = E;
    const int gmax = max_resident(fn, smem_bytes(probe));
    if (gmax < 1)
        return false;
    const int64_t units = static_cast<int64_t>(T) * (fp8 ? H / 16 : H / 8);
    g = make_geom(T, k, E, R, gmax, units);
    return true;
}

}  // namespace

size_t route_dispatch_workspace_bytes(int T, int k, int E, int R)
{
    // Sized for the most CTAs any variant of the kernel can keep resident
    // (2048 threads per SM / 512): the chunk count only grows with the grid,
    // so every launch's geometry fits.
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm < 1)
        return 0;
    const FusedGeom g = make_geom(T, k, E, R, nsm * (2048 / kThreads), 0);
    return (ws_layout(g).total * sizeof(int32_t) + 255) / 256 * 256;
}

cudaError_t route_dispatch(const float *logits, int T, int E, int k, int renormalize, int R,
                           int capacity, const uint16_t *x, int H, bool fp8, int32_t *topk_idx,
                           float *topk_w, int32_t *expert_counts, int32_t *expert_src_counts,
                           int32_t *rank_counts, int32_t *expert_offsets, int32_t *dispatch_pos,
                           int32_t *recv_src, void *recv, float *recv_scale, int64_t rows,
                           void *workspace, size_t ws_bytes, int32_t *dev_status, cudaStream_t s,
                           bool *ws_too_small, const RouteEx *ex)
{
    FusedGeom g;
    KernelFn fn;
    *ws_too_small = false;
    const int kk = k + (ex ? ex->n_shared : 0);   // slots per token
    const int El = ex ? ex->E_phys : E;           // the layout's experts
    if (!device_geom(T, kk, El, R, H, fp8, E, g, fn))
        return cudaErrorInvalidConfiguration;
    if (ws_bytes < ws_layout(g).total * sizeof(int32_t)) {
        *ws_too_small = true;
        return cudaSuccess;
    }
    FusedArgs a;
    a.logits = logits;
    a.El = E;
    a.kr = k;
    a.renormalize = renormalize;
    a.ex_on = ex ? 1 : 0;
    a.shared_weight = ex ? ex->shared_weight : 1.0f;
    a.replica_offsets = ex ? ex->replica_offsets : nullptr;
    a.replica_ids = ex ? ex->replica_ids : nullptr;
    a.n_replica_ids = ex ? ex->n_replica_ids : 0;
    a.x = reinterpret_cast<const uint4 *>(x);
    a.H = H;
    a.capacity = capacity;
    a.rows = rows;
    a.topk_idx = topk_idx;
    a.topk_w = topk_w;
    a.expert_counts = expert_counts;
    a.expert_src_counts = expert_src_counts;
    a.rank_counts = rank_counts;
    a.expert_offsets = expert_offsets;
    a.dispatch_pos = dispatch_pos;
    a.recv_src = recv_src;
    a.recv = recv;
    a.recv_scale = recv_scale;
    a.ws = static_cast<int32_t *>(workspace);
    a.dev_status = dev_status;

    const size_t smem = smem_bytes(g);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g.G);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fn, a, g);
}

}  // namespace moe
