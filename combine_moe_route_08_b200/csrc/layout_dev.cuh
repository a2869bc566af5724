// layout_dev.cuh -- device pieces of the deterministic layout, shared by the
// layout kernels and the fused route -> layout -> dispatch kernel.
//
// Within a chunk of consecutive slots, each warp owns a contiguous run of
// 32-slot steps.  A slot's position inside its expert is
//   (slots of the expert in earlier chunks) + (in earlier warps of the chunk)
//   + (in earlier steps of the warp) + (in lower lanes of the same step),
// so every position comes from counts and prefix sums; atomics never decide
// an order.
//
// The equality mask of a warp step ("which lanes hold my expert") is built
// from one __ballot_sync per key bit; __match_any_sync would give the same
// mask but costs about 2000 cycles per call on this part (measured with
// clock64 stamps).
#pragma once

#include "common.cuh"

namespace moe {

__device__ __forceinline__ unsigned lanemask_lt()
{
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Lanes of the warp holding the same key as this lane: a lane matches where
// every key bit agrees.
__device__ __forceinline__ unsigned match_mask(int key, int nbits)
{
    unsigned mask = kFullMask;
    for (int b = 0; b < nbits; ++b) {
        const bool bit = (key >> b) & 1;
        const unsigned bal = __ballot_sync(kFullMask, bit);
        mask &= bit ? bal : ~bal;
    }
    return mask;
}

// Key bits: enough for max(E - 1, 31), plus one bit that marks a slot that
// is empty, masked or invalid (key = lane | that bit, unique in the warp).
__device__ __forceinline__ int key_bits(int E)
{
    return 32 - __clz(max(E - 1, 31)) + 1;
}

__device__ __forceinline__ int match_key(int e, int E, int lane, int nbits)
{
    return (static_cast<unsigned>(e) < static_cast<unsigned>(E)) ? e : (lane | (1 << (nbits - 1)));
}

// Count the warp run's slots per expert into the warp's private row `mywh`
// with one add per distinct expert of a step, by its lowest lane (no
// atomics; the equality masks cost more instructions than warp_count's
// atomics but fewer registers, which the fused kernel's budget needs).
template <int MAXS>
__device__ __forceinline__ void warp_histogram(const int (&e)[MAXS], int64_t w0, int64_t w1, int E,
                                               int nb, int32_t *mywh)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int s = 0; s < MAXS; ++s) {
        if (w0 + 32 * s >= w1)
            break;  // warp-uniform
        const bool valid = static_cast<unsigned>(e[s]) < static_cast<unsigned>(E);
        const unsigned mask = match_mask(match_key(e[s], E, lane, nb), nb);
        if (valid && lane == __ffs(mask) - 1)
            mywh[e[s]] += __popc(mask);
        __syncwarp();
    }
}

// Count the warp run's slots per expert into the warp's private row `mywh`
// with one shared-memory atomic per slot: counts do not depend on the order
// in which they are added, so atomics are safe here (unlike positions).
template <int MAXS>
__device__ __forceinline__ void warp_count(const int (&e)[MAXS], int64_t w0, int64_t w1, int E,
                                           int32_t *mywh)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int s = 0; s < MAXS; ++s)
        if (w0 + 32 * s + lane < w1 && static_cast<unsigned>(e[s]) < static_cast<unsigned>(E))
            atomicAdd(mywh + e[s], 1);
}

// Turn the per-warp rows wh[NW][E] into per-warp bases: chb[x] (slots of x
// in earlier chunks) plus the counts of the earlier warps.  The whole CTA of
// NW warps takes part: G adjacent lanes per expert (G a power of two, G * E
// <= NW * 32 when it can be above 1) each sum the counts of NW / G
// consecutive warps, scan their G partial sums by shuffles, then rewrite
// their warps' rows as running bases (chains G times shorter than one thread
// per expert walking all NW rows).  Called by every thread.
template <int NW>
__device__ __forceinline__ void warp_bases_par(int32_t *wh, const int32_t *chb, int E)
{
    int G = 1;
    while (2 * G <= NW && 2 * G * E <= NW * 32)
        G *= 2;
    const int per = NW / G;
    // whole warps (every lane takes part in the shuffles); more than one pass
    // only when E exceeds the CTA's threads (then G = 1)
    const int span = (E * G + 31) / 32 * 32;
    for (int idx = threadIdx.x; idx < span; idx += NW * 32) {
        const int x = idx / G, part = idx % G;
        const bool valid = x < E;
        int sum = 0;
        if (valid)
            for (int ww = part * per; ww < (part + 1) * per; ++ww)
                sum += wh[ww * E + x];
        int incl = sum;
        for (int o = 1; o < G; o <<= 1) {
            const int t = __shfl_up_sync(kFullMask, incl, o, G);
            if (part >= o)
                incl += t;
        }
        if (valid) {
            int run = chb[x] + incl - sum;
            for (int ww = part * per; ww < (part + 1) * per; ++ww) {
                const int t = wh[ww * E + x];
                wh[ww * E + x] = run;
                run += t;
            }
        }
    }
}

// Position of this lane's slot among the equal experts of its warp, given the
// warp's running bases `mywh` (advanced past this step on return).  Returns 0
// for an invalid slot.  Called by all 32 lanes.
__device__ __forceinline__ int rank_step(int e, int E, int nb, int32_t *mywh)
{
    const int lane = threadIdx.x & 31;
    const bool valid = static_cast<unsigned>(e) < static_cast<unsigned>(E);
    const unsigned mask = match_mask(match_key(e, E, lane, nb), nb);
    const int p = valid ? mywh[e] + __popc(mask & lanemask_lt()) : 0;
    __syncwarp();
    if (valid && lane == __ffs(mask) - 1)
        mywh[e] += __popc(mask);
    __syncwarp();
    return p;
}

// In-place exclusive scan of a[0..n) by a CTA of NW warps, in tiles of
// NW * 32 elements with a running carry; a[n] receives the total.  `tot` is
// NW + 1 ints of shared scratch.  Called by every thread of the CTA.
template <int NW>
__device__ void block_exclusive_scan(int32_t *a, int n, int32_t *tot)
{
    static_assert(NW <= 32, "one warp scans the warp totals");
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    int carry = 0;
    for (int base = 0; base < n; base += NW * 32) {
        const int i = base + tid;
        const int v = (i < n) ? a[i] : 0;
        int incl = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int t = __shfl_up_sync(kFullMask, incl, off);
            if (lane >= off)
                incl += t;
        }
        if (lane == 31)
            tot[w] = incl;
        __syncthreads();
        if (w == 0) {
            const int t = (lane < NW) ? tot[lane] : 0;
            int x = t;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(kFullMask, x, off);
                if (lane >= off)
                    x += y;
            }
            if (lane < NW)
                tot[lane] = x - t;  // exclusive over warps
            if (lane == NW - 1)
                tot[NW] = x;
        }
        __syncthreads();
        if (i < n)
            a[i] = carry + tot[w] + incl - v;
        carry += tot[NW];
        __syncthreads();  // tot is rewritten by the next tile
    }
    if (tid == 0)
        a[n] = carry;
    __syncthreads();
}

}  // namespace moe
