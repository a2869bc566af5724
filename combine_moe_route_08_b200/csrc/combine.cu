// combine.cu -- gather each token's k expert rows and form the router-
// weighted sum in fp32, stored as bf16.  The rows arrive as bf16, or as E4M3
// codes with 1x128 fp32 scales (the dispatch format used for the way back).
//
// "Efficient and portable mixture-of-experts communication", "Combinação":
// the receiver reads the routing table to know which buffer to read and which
// weight each expert contribution gets, and computes their weighted sum;
// "Enabling trillion-parameter models on AWS EFA", "Dağıtım/Birleştirme
// Gecikmesi": bf16 combine, accumulation only at the receiver.
//
// bf16 rows: one CTA per token; a thread owns 8 consecutive channels (16
// bytes of each row), or, for long combines with 32-byte aligned buffers, 16
// channels read 32 bytes at a time.  FP8 rows: a persistent grid walking the
// tokens, a thread owning 16 channels.  Either way the token's row indices and weights
// are held in registers, so all k (up to 8) 16-byte loads of a pass issue
// back to back before any is used; then the sum runs in ascending j with a
// separate binary32 multiply and add per term (__fmul_rn / __fadd_rn are
// never contracted into an FMA), so the output is bit-reproducible.
#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kMaxThreads = 512;
// FP8 combine: at most 448 threads per CTA (one pass at H = 7168) so that two
// CTAs fit on an SM with 72 registers per thread, enough to hold 8 rows of 16
// codes in flight without spilling.
constexpr int kFp8Threads = 448;
// Rows read (T * k * H * 2 bytes) from which the bf16 combine takes the
// 32-byte-load form (k_combine_bf16_w32): between the measured sizes where it
// lost (0.7 GB) or tied (0.9 GB) and the one where it won (3.8 GB).
constexpr int64_t kLongCombineBytes = int64_t(2) << 30;

// Lane j of every warp loads the token's j-th row index and weight (no
// shared memory, no CTA barrier: each warp starts its row loads as soon as its
// own index load returns); the first KREG are broadcast into registers by
// shuffles, so the loads of a pass are issued back to back, and terms beyond
// KREG follow in order, broadcast the same way.  Passes are CTA-uniform so
// every lane takes part in the shuffles.  (Against the shared-memory version:
// 77.0 against 77.8 us alone at dsv3, 1092 against 1105 us for the prefill
// step; outputs identical.)
template <int KREG>
__global__ void __launch_bounds__(kMaxThreads)
    k_combine_bf16(const uint4 *__restrict__ y, const int32_t *__restrict__ dispatch_pos,
                   const float *__restrict__ topk_w, int nvec, int k, int64_t rows,
                   uint4 *__restrict__ out, int32_t *__restrict__ dev_status)
{
    const int g = blockIdx.x;
    const int lane = threadIdx.x & 31;
    pdl_wait();
    int myr = -1;
    float myw = 0.0f;
    if (lane < k) {
        myr = __ldg(dispatch_pos + static_cast<size_t>(g) * k + lane);
        myw = __ldg(topk_w + static_cast<size_t>(g) * k + lane);
        if (myr < -1 || myr >= rows) {
            if (threadIdx.x < 32)
                report(dev_status, MOE_ERR_INVALID_ARG);
            myr = -1;
        }
    }
    int rr[KREG];
    float ww[KREG];
#pragma unroll
    for (int j = 0; j < KREG; ++j) {
        rr[j] = __shfl_sync(kFullMask, myr, j);
        ww[j] = __shfl_sync(kFullMask, myw, j);
    }

    for (int v0 = 0; v0 < nvec; v0 += blockDim.x) {  // CTA-uniform trips (shuffles)
        const int v = v0 + threadIdx.x;
        const bool act = v < nvec;
        float acc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
            acc[c] = 0.0f;
        uint4 d[KREG];
#pragma unroll
        for (int j = 0; j < KREG; ++j)
            d[j] = (act && rr[j] >= 0) ? ld_stream_v4(y + static_cast<size_t>(rr[j]) * nvec + v)
                                       : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int j = 0; j < KREG; ++j) {
            if (rr[j] >= 0) {
                const uint32_t wds[4] = {d[j].x, d[j].y, d[j].z, d[j].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(ww[j], bf16_lo(wds[i])));
                    acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __fmul_rn(ww[j], bf16_hi(wds[i])));
                }
            }
        }
        // k > KREG: the remaining terms, in order, each row index and weight
        // broadcast from its lane by a shuffle
        for (int j = KREG; j < k; ++j) {
            const int r = __shfl_sync(kFullMask, myr, j);
            const float wj = __shfl_sync(kFullMask, myw, j);
            if (!act || r < 0)
                continue;
            const uint4 e = ld_stream_v4(y + static_cast<size_t>(r) * nvec + v);
            const uint32_t wds[4] = {e.x, e.y, e.z, e.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(wj, bf16_lo(wds[i])));
                acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __fmul_rn(wj, bf16_hi(wds[i])));
            }
        }
        const uint4 o = make_uint4(bf16x2_rn(acc[0], acc[1]), bf16x2_rn(acc[2], acc[3]),
                                   bf16x2_rn(acc[4], acc[5]), bf16x2_rn(acc[6], acc[7]));
        if (act)
            st_stream_v4(out + static_cast<size_t>(g) * nvec + v, o);
    }
    pdl_trigger();
}

// Two E4M3 codes (low byte first) -> two binary32 values.  The hardware
// converts E4M3 to binary16, which holds every E4M3 value (subnormals, +-448,
// NaN) exactly, and binary16 -> binary32 is exact, so the decode is exact.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t two_codes)
{
    const __half2_raw raw =
        __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_codes), __NV_E4M3);
    return __half22float2(*reinterpret_cast<const __half2 *>(&raw));
}

// Packed binary32 multiply (sm_100): each lane is one IEEE product rounded to
// nearest even, exactly as __fmul_rn, at half the instructions.  Only
// multiplies are packed: ptxas was measured to fuse a packed multiply and a
// following packed add (add.rn.f32x2) into a fused multiply-add, which
// changes the rounding, whereas it keeps a scalar __fadd_rn of a packed
// product separate (probe over 8.4 M random triples: 0 differences against
// scalar ops, against 3.7 M with packed adds).
__device__ __forceinline__ float2 fmul2_rn(float2 a, float2 b)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// One product per element restores the expert row, v = decode(q) * s; then the
// same ascending-j sum of w_j * v as the bf16 combine.  Both products run two
// channels per packed instruction; the sums are scalar.  A thread owns 16
// channels (16 codes of each row, inside one 128-channel block, so one scale
// per row), summed in two halves of 8, and writes 32 bytes of bf16.
//
// Persistent grid: as many CTAs as fit on the device at once walk the tokens
// round-robin (token g, g + gridDim.x, ...).  Lane j of every warp holds the
// token's j-th row index and weight (shuffled to the others, no shared
// memory, no CTA barrier) and loads the NEXT token's while the current one
// is summed, so the index round trip leaves the critical path and no wave
// of CTAs runs half empty.  Kernel alone, bit-identical outputs: dsv3 59.5 ->
// 57.5 us, prefill 426.5 -> 417.0 us against a CTA per four (eight) tokens
// with their indices staged in shared memory.
template <int KREG, bool EXACT>
__global__ void __launch_bounds__(kFp8Threads, KREG <= 9 ? 2 : 1)
    k_combine_fp8(const uint4 *__restrict__ yq, const float *__restrict__ ys,
                  const int32_t *__restrict__ dispatch_pos, const float *__restrict__ topk_w, int T,
                  int H, int k, int64_t rows, uint4 *__restrict__ out,
                  int32_t *__restrict__ dev_status)
{
    const int lane = threadIdx.x & 31;
    const int ngrp = H / 16, S = H / 128;
    // lane j < k: row index and weight of slot j of token g (-1: skipped)
    auto fetch = [&](int g, int &r, float &wv) {
        r = -1;
        wv = 0.0f;
        if (g < T && lane < k) {
            r = __ldg(dispatch_pos + static_cast<size_t>(g) * k + lane);
            wv = __ldg(topk_w + static_cast<size_t>(g) * k + lane);
            if (r < -1 || r >= rows) {
                if (threadIdx.x < 32)
                    report(dev_status, MOE_ERR_INVALID_ARG);
                r = -1;
            }
        }
    };
    pdl_wait();
    int myr;
    float myw;
    fetch(blockIdx.x, myr, myw);

    // adds row j's 8 channels held in words (w0, w1) to acc
    auto add_half = [&](float (&acc)[8], uint32_t w0, uint32_t w1, float sc, float wj) {
        const float2 s2 = make_float2(sc, sc), ww = make_float2(wj, wj);
        const uint32_t wds[2] = {w0, w1};
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float2 plo = fmul2_rn(ww, fmul2_rn(e4m3x2_to_float2(wds[i] & 0xffffu), s2));
            const float2 phi = fmul2_rn(ww, fmul2_rn(e4m3x2_to_float2(wds[i] >> 16), s2));
            acc[4 * i] = __fadd_rn(acc[4 * i], plo.x);
            acc[4 * i + 1] = __fadd_rn(acc[4 * i + 1], plo.y);
            acc[4 * i + 2] = __fadd_rn(acc[4 * i + 2], phi.x);
            acc[4 * i + 3] = __fadd_rn(acc[4 * i + 3], phi.y);
        }
    };

    for (int g = blockIdx.x; g < T; g += gridDim.x) {  // CTA-uniform
        int nr;
        float nw;
        fetch(g + gridDim.x, nr, nw);  // the next token's, in flight during this one
        int rr[KREG];
#pragma unroll
        for (int j = 0; j < KREG; ++j)
            rr[j] = __shfl_sync(kFullMask, myr, j);  // lanes >= k hold -1
        // EXACT: one pass with every thread owning a unit (H / 16 == blockDim.x)
        // and exactly KREG slots per token, so no guards and no tail
        for (int t0 = 0; t0 < ngrp; t0 += blockDim.x) {  // CTA-uniform trips (shuffles)
            const int t = t0 + threadIdx.x;
            const bool act = EXACT || t < ngrp;
            uint4 d[KREG];
            float sc[KREG];
#pragma unroll
            for (int j = 0; j < KREG; ++j) {
                d[j] = make_uint4(0, 0, 0, 0);
                sc[j] = 0.0f;
                if (act && rr[j] >= 0) {
                    d[j] = ld_stream_v4(yq + static_cast<size_t>(rr[j]) * ngrp + t);
                    sc[j] = __ldg(ys + static_cast<size_t>(rr[j]) * S + (t >> 3));
                }
            }
            uint4 *o = out + static_cast<size_t>(g) * (H / 8) + 2 * t;
            // channels 16t .. 16t+7 from words x, y; then 16t+8 .. 16t+15 from z, w
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float acc[8];
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    acc[c] = 0.0f;
#pragma unroll
                for (int j = 0; j < KREG; ++j) {
                    const float wj = __shfl_sync(kFullMask, myw, j);
                    if (rr[j] >= 0)
                        add_half(acc, half ? d[j].z : d[j].x, half ? d[j].w : d[j].y, sc[j], wj);
                }
                for (int j = KREG; !EXACT && j < k; ++j) {  // k > KREG: the rest, in order
                    const int r = __shfl_sync(kFullMask, myr, j);
                    const float wj = __shfl_sync(kFullMask, myw, j);
                    if (!act || r < 0)
                        continue;
                    const uint4 e = ld_stream_v4(yq + static_cast<size_t>(r) * ngrp + t);
                    add_half(acc, half ? e.z : e.x, half ? e.w : e.y,
                             __ldg(ys + static_cast<size_t>(r) * S + (t >> 3)), wj);
                }
                if (act)
                    st_stream_v4(o + half,
                                 make_uint4(bf16x2_rn(acc[0], acc[1]), bf16x2_rn(acc[2], acc[3]),
                                            bf16x2_rn(acc[4], acc[5]), bf16x2_rn(acc[6], acc[7])));
            }
            if (EXACT)
                break;
        }
        myr = nr;
        myw = nw;
    }
    pdl_trigger();
}

// 32 bytes of a row in one load (sm_100's 256-bit vector load), bypassing L1.
struct Words8 {
    uint32_t w[8];
};
__device__ __forceinline__ Words8 ld_stream_v8(const void *p)
{
    Words8 v;
    asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]), "=r"(v.w[4]),
                   "=r"(v.w[5]), "=r"(v.w[6]), "=r"(v.w[7])
                 : "l"(p));
    return v;
}

// The bf16 combine for long combines (k <= 8, H % 16 == 0, y and out 32-byte
// aligned): a thread owns 16 channels, reads 32 bytes of a row per load and
// takes the rows two at a time (40 registers, three CTAs per SM); the same
// products and sums in the same order as k_combine_bf16, so the same bits.
// Kernel alone and in whole steps, alternating, at T = 32768, H = 7168,
// k = 8: 605.5 against 624.9 us, steps 1052.5 against 1075.5 us.  In the
// decode chains (4096 and 6144 tokens) it made whole steps slower (153.1
// against 147.3, 218.5 against 215.0 us) with the kernel alone unchanged, so
// it is used only when the rows read reach kLongCombineBytes.
__global__ void __launch_bounds__(kMaxThreads, 3)
    k_combine_bf16_w32(const uint8_t *__restrict__ y, const int32_t *__restrict__ dispatch_pos,
                       const float *__restrict__ topk_w, int nu, int k, int64_t rows,
                       uint4 *__restrict__ out, int32_t *__restrict__ dev_status)
{
    const int g = blockIdx.x;
    const int lane = threadIdx.x & 31;
    pdl_wait();
    int myr = -1;
    float myw = 0.0f;
    if (lane < k) {
        myr = __ldg(dispatch_pos + static_cast<size_t>(g) * k + lane);
        myw = __ldg(topk_w + static_cast<size_t>(g) * k + lane);
        if (myr < -1 || myr >= rows) {
            if (threadIdx.x < 32)
                report(dev_status, MOE_ERR_INVALID_ARG);
            myr = -1;
        }
    }
    int rr[8];
    float ww[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {  // lanes >= k hold -1
        rr[j] = __shfl_sync(kFullMask, myr, j);
        ww[j] = __shfl_sync(kFullMask, myw, j);
    }
    for (int v0 = 0; v0 < nu; v0 += blockDim.x) {  // CTA-uniform trips (shuffles)
        const int v = v0 + threadIdx.x;
        const bool act = v < nu;
        float acc[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
            acc[c] = 0.0f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // rows 2q and 2q + 1
            Words8 d[2];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int j = 2 * q + jj;
                if (act && rr[j] >= 0) {
                    d[jj] = ld_stream_v8(y + (static_cast<size_t>(rr[j]) * nu + v) * 32);
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        d[jj].w[i] = 0u;
                }
            }
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int j = 2 * q + jj;
                if (rr[j] >= 0) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(ww[j], bf16_lo(d[jj].w[i])));
                        acc[2 * i + 1] =
                            __fadd_rn(acc[2 * i + 1], __fmul_rn(ww[j], bf16_hi(d[jj].w[i])));
                    }
                }
            }
        }
        if (act) {
            uint4 *o = out + static_cast<size_t>(g) * (2 * nu) + 2 * v;
            st_stream_v4(o, make_uint4(bf16x2_rn(acc[0], acc[1]), bf16x2_rn(acc[2], acc[3]),
                                       bf16x2_rn(acc[4], acc[5]), bf16x2_rn(acc[6], acc[7])));
            st_stream_v4(o + 1, make_uint4(bf16x2_rn(acc[8], acc[9]), bf16x2_rn(acc[10], acc[11]),
                                           bf16x2_rn(acc[12], acc[13]),
                                           bf16x2_rn(acc[14], acc[15])));
        }
    }
    pdl_trigger();
}

int threads_for(int units, int max_threads = kMaxThreads)
{
    const int passes = ceil_div(units, max_threads);
    return round_up(ceil_div(units, passes), 32);
}

}  // namespace

namespace {

// CTAs of k_combine_fp8<KREG, EXACT> resident at once on the current device
// (the persistent grid), for `threads` threads per CTA; remembered per device.
template <int KREG, bool EXACT>
int fp8_grid(int threads)
{
    constexpr int kMaxDev = 64;  // devices whose answer is remembered; others ask each time
    static std::atomic<int> cache[kMaxDev][kFp8Threads / 32 + 1];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0)
        return 0;
    std::atomic<int> *slot = (dev < kMaxDev) ? &cache[dev][threads / 32] : nullptr;
    int v = slot ? slot->load(std::memory_order_relaxed) : 0;
    if (v > 0)
        return v;
    int nsm = 0, per = 0;
    if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, k_combine_fp8<KREG, EXACT>, threads, 0) !=
            cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    v = std::max(1, nsm * per);
    if (slot)
        slot->store(v, std::memory_order_relaxed);
    return v;
}

template <int KREG, bool EXACT>
cudaError_t launch_fp8(const uint8_t *yq, const float *ys, const int32_t *dispatch_pos,
                       const float *topk_w, int T, int H, int k, int64_t rows, uint16_t *out,
                       int32_t *dev_status, cudaStream_t s)
{
    const int threads = threads_for(H / 16, kFp8Threads);
    const int resident = fp8_grid<KREG, EXACT>(threads);
    if (resident < 1)
        return cudaErrorInvalidConfiguration;
    const int grid = std::min(T, resident);
    return launch_pdl(k_combine_fp8<KREG, EXACT>, dim3(grid), dim3(threads), 0, s,
                      reinterpret_cast<const uint4 *>(yq), ys, dispatch_pos, topk_w, T, H, k, rows,
                      reinterpret_cast<uint4 *>(out), dev_status);
}

}  // namespace

cudaError_t combine_fp8(const uint8_t *yq, const float *ys, const int32_t *dispatch_pos,
                        const float *topk_w, int T, int H, int k, int64_t rows, uint16_t *out,
                        int32_t *dev_status, cudaStream_t s)
{
    // k = 8 with H / 16 a whole multiple of 32 up to 448 units (one pass of
    // full warps, every thread busy; H = 7168 among them): the exact form.
    // Bit-identical to the general one and faster, in 10-step graphs at
    // H = 7168: 4096 tokens 60.3 against 63.5 us, 6144 tokens 91.4 against
    // 96.1, 32768 tokens 482.6 against 516.9.
    const int ngrp = H / 16;
    if (k == 8 && ngrp % 32 == 0 && ngrp <= kFp8Threads)
        return launch_fp8<8, true>(yq, ys, dispatch_pos, topk_w, T, H, k, rows, out, dev_status, s);
    if (k <= 2)
        return launch_fp8<2, false>(yq, ys, dispatch_pos, topk_w, T, H, k, rows, out, dev_status, s);
    if (k <= 4)
        return launch_fp8<4, false>(yq, ys, dispatch_pos, topk_w, T, H, k, rows, out, dev_status, s);
    if (k <= 8)
        return launch_fp8<8, false>(yq, ys, dispatch_pos, topk_w, T, H, k, rows, out, dev_status, s);
    if (k == 9)
        return launch_fp8<9, false>(yq, ys, dispatch_pos, topk_w, T, H, k, rows, out, dev_status, s);
    return launch_fp8<16, false>(yq, ys, dispatch_pos, topk_w, T, H, k, rows, out, dev_status, s);
}

bool combine_bf16_long_form(int T, int H, int k)
{
    return k <= 8 && H % 16 == 0 && static_cast<int64_t>(T) * k * H * 2 >= kLongCombineBytes;
}

cudaError_t combine_bf16(const uint16_t *y, const int32_t *dispatch_pos, const float *topk_w,
                         int T, int H, int k, int64_t rows, uint16_t *out, int32_t *dev_status,
                         cudaStream_t s)
{
    const int nvec = H / 8;
    const dim3 grid(T), block(threads_for(nvec));
    const uint4 *yv = reinterpret_cast<const uint4 *>(y);
    uint4 *ov = reinterpret_cast<uint4 *>(out);
    if (combine_bf16_long_form(T, H, k) && reinterpret_cast<uintptr_t>(y) % 32 == 0 &&
        reinterpret_cast<uintptr_t>(out) % 32 == 0)
        return launch_pdl(k_combine_bf16_w32, grid, dim3(threads_for(H / 16)), 0, s,
                          reinterpret_cast<const uint8_t *>(y), dispatch_pos, topk_w, H / 16, k,
                          rows, ov, dev_status);
    if (k <= 2)
        return launch_pdl(k_combine_bf16<2>, grid, block, 0, s, yv, dispatch_pos, topk_w, nvec, k,
                          rows, ov, dev_status);
    if (k <= 4)
        return launch_pdl(k_combine_bf16<4>, grid, block, 0, s, yv, dispatch_pos, topk_w, nvec, k,
                          rows, ov, dev_status);
    if (k <= 8)
        return launch_pdl(k_combine_bf16<8>, grid, block, 0, s, yv, dispatch_pos, topk_w, nvec, k,
                          rows, ov, dev_status);
    if (k == 9)  // eight routed experts and a shared one
        return launch_pdl(k_combine_bf16<9>, grid, block, 0, s, yv, dispatch_pos, topk_w, nvec, k,
                          rows, ov, dev_status);
    return launch_pdl(k_combine_bf16<16>, grid, block, 0, s, yv, dispatch_pos, topk_w, nvec, k,
                      rows, ov, dev_status);
}

}  // namespace moe
