// dispatch.cu -- row scatter of each token into its k expert rows, as bf16 or
// as OCP E4M3 with 1x128 fp32 block scales.
//
// "Enabling trillion-parameter models on AWS EFA", "Dağıtım ve Birleştirme":
// tokens are packed into contiguous per-expert buffers at the offsets the
// counts gave; "Dağıtım/Birleştirme Gecikmesi": block-scaled fp8 dispatch.
// DeepSeek-V3 fragments: activations scaled per token per 128 channels, and
// the wish to fuse the fp8 cast into the load from global memory -- here the
// cast happens in registers between the single read of x and the k writes.
//
// One CTA per token: the row of x is read once (16-byte loads that skip L1),
// quantised once, and written k times with 16-byte streaming stores, each
// destination row by the whole CTA in one coalesced sweep.  Before waiting
// for the layout, the first CTAs prefetch x into L2 (prefetch_x) so that its
// HBM read overlaps the latency-bound route and layout.
#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "dispatch_dev.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kMaxK = 32;
constexpr int kMaxThreads = 512;

// The first pf_ctas CTAs start moving the first pf_bytes of x from HBM into
// L2 before they wait for the layout (l2_prefetch_share).  With the route and
// layout kernels releasing their dependents at their start, these CTAs are
// resident while those latency-bound kernels leave HBM almost idle, so x
// (58.7 MB at T = 4096, H = 7168) is read during the layout and the dispatch
// proper is bound by its writes.
__device__ __forceinline__ void prefetch_x(const void *x, int64_t pf_bytes, int pf_ctas)
{
    const int P = min(static_cast<int>(gridDim.x), pf_ctas);
    if (static_cast<int>(blockIdx.x) < P)
        l2_prefetch_share(x, pf_bytes, blockIdx.x, P);
}

// Load the token's k destination rows into shared memory; rows outside
// [0, rows) other than -1 are reported and skipped.
__device__ __forceinline__ void load_rows(const int32_t *__restrict__ dispatch_pos, int g, int k,
                                          int64_t rows, int32_t *srow, int32_t *dev_status)
{
    pdl_wait();
    if (threadIdx.x < k) {
        int r = dispatch_pos[static_cast<size_t>(g) * k + threadIdx.x];
        if (r < -1 || r >= rows) {
            report(dev_status, MOE_ERR_INVALID_ARG);
            r = -1;
        }
        srow[threadIdx.x] = r;
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kMaxThreads)
    k_dispatch_bf16(const uint4 *__restrict__ x, int nvec, int k,
                    const int32_t *__restrict__ dispatch_pos, uint4 *__restrict__ recv_x,
                    int64_t rows, int32_t *__restrict__ dev_status, int64_t pf_bytes,
                    int pf_ctas)
{
    __shared__ int32_t srow[kMaxK];
    const int g = blockIdx.x;
    prefetch_x(x, pf_bytes, pf_ctas);
    load_rows(dispatch_pos, g, k, rows, srow, dev_status);
    const uint4 *xr = x + static_cast<size_t>(g) * nvec;
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
        const uint4 d = ld_stream_v4(xr + v);
        for (int j = 0; j < k; ++j) {
            const int r = srow[j];
            if (r >= 0)
                st_stream_v4(recv_x + static_cast<size_t>(r) * nvec + v, d);
        }
    }
    pdl_trigger();
}

// Thread t of the token owns channels [16t, 16t + 16) (quant_e4m3_x16).
// Scales go to recv_scale[r * S + b] (row-major) or, with scale_ld > 0, to
// recv_scale[b * scale_ld + r] (column-major: each 128-channel block's scales
// contiguous over the rows, the operand layout of a grouped FP8 GEMM).
__global__ void __launch_bounds__(kMaxThreads)
    k_dispatch_fp8(const uint4 *__restrict__ x, int H, int k,
                   const int32_t *__restrict__ dispatch_pos, uint8_t *__restrict__ recv_q,
                   float *__restrict__ recv_scale, int64_t rows, int64_t scale_ld,
                   int32_t *__restrict__ dev_status, int64_t pf_bytes, int pf_ctas)
{
    __shared__ int32_t srow[kMaxK];
    const int g = blockIdx.x;
    prefetch_x(x, pf_bytes, pf_ctas);
    load_rows(dispatch_pos, g, k, rows, srow, dev_status);
    const int ngrp = H / 16;
    const int S = H / 128;
    const uint4 *xr = x + static_cast<size_t>(g) * (H / 8);

    for (int t0 = 0; t0 < ngrp; t0 += blockDim.x) {  // CTA-uniform trips (shuffles)
        const int t = t0 + threadIdx.x;
        const bool act = t < ngrp;
        uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
        if (act) {
            a = ld_stream_v4(xr + 2 * t);
            b = ld_stream_v4(xr + 2 * t + 1);
        }
        float s;
        const uint4 q = quant_e4m3_x16(a, b, s);
        if (act) {
            for (int j = 0; j < k; ++j) {
                const int r = srow[j];
                if (r < 0)
                    continue;
                st_stream_v4(recv_q + static_cast<size_t>(r) * H + 16 * t, q);
                if ((t & 7) == 0) {
                    const size_t at = (scale_ld > 0)
                                          ? static_cast<size_t>(t >> 3) * scale_ld + r
                                          : static_cast<size_t>(r) * S + (t >> 3);
                    __stcs(recv_scale + at, s);
                }
            }
        }
    }
    pdl_trigger();
}

// 32 bytes in one streaming store (sm_100's 256-bit vector store).
__device__ __forceinline__ void st_stream_v8(void *p, uint4 a, uint4 b)
{
    asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p),
                 "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
                 : "memory");
}

// The FP8 dispatch when x is read from HBM (too large to be prefetched into
// L2; H % 256 == 0, recv_q 32-byte aligned): thread t owns channels
// [32t, 32t + 32) (quant_e4m3_x32) and writes each row's 32 codes with one
// 256-bit store.  The same codes and scales as k_dispatch_fp8.  Alternating,
// graphs of 10, at T = 32768, H = 7168, k = 8: the kernel 381.2 against
// 401.5 us, whole steps 1039.4 against 1056.2 us.  With x prefetched into L2
// (T = 4096 and 6144) it was slower (54.0 against 51.1 us at T = 4096) and
// is not used there.
__global__ void __launch_bounds__(kMaxThreads)
    k_dispatch_fp8_w32(const uint4 *__restrict__ x, int H, int k,
                       const int32_t *__restrict__ dispatch_pos, uint8_t *__restrict__ recv_q,
                       float *__restrict__ recv_scale, int64_t rows, int64_t scale_ld,
                       int32_t *__restrict__ dev_status)
{
    __shared__ int32_t srow[kMaxK];
    const int g = blockIdx.x;
    load_rows(dispatch_pos, g, k, rows, srow, dev_status);
    const int nu = H / 32;
    const int S = H / 128;
    const uint4 *xr = x + static_cast<size_t>(g) * (H / 8);
    for (int t0 = 0; t0 < nu; t0 += blockDim.x) {  // CTA-uniform trips (shuffles)
        const int t = t0 + threadIdx.x;
        const bool act = t < nu;
        uint4 in[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            in[u] = act ? ld_stream_v4(xr + 4 * t + u) : make_uint4(0, 0, 0, 0);
        float s;
        uint4 q0, q1;
        quant_e4m3_x32(in, q0, q1, s);
        if (act) {
            for (int j = 0; j < k; ++j) {
                const int r = srow[j];
                if (r < 0)
                    continue;
                st_stream_v8(recv_q + static_cast<size_t>(r) * H + 32 * t, q0, q1);
                if ((t & 3) == 0) {
                    const size_t at = (scale_ld > 0)
                                          ? static_cast<size_t>(t >> 2) * scale_ld + r
                                          : static_cast<size_t>(r) * S + (t >> 2);
                    __stcs(recv_scale + at, s);
                }
            }
        }
    }
    pdl_trigger();
}

__global__ void k_quantize_e4m3(const float *__restrict__ v, int64_t n, uint8_t *__restrict__ q)
{
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t p = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; 2 * p < n; p += stride) {
        const int64_t i = 2 * p;
        if (i + 1 < n) {
            const uint32_t c = e4m3x2(v[i], v[i + 1]);
            q[i] = static_cast<uint8_t>(c & 0xff);
            q[i + 1] = static_cast<uint8_t>(c >> 8);
        } else {
            q[i] = static_cast<uint8_t>(e4m3x2(v[i], 0.0f) & 0xff);
        }
    }
}

int threads_for(int units)
{
    // fewest passes of at most kMaxThreads threads, then as few threads as
    // cover the units in that many passes (a multiple of the warp size)
    const int passes = ceil_div(units, kMaxThreads);
    return round_up(ceil_div(units, passes), 32);
}

}  // namespace

// How much of x (x_bytes, a multiple of 16) the dispatch prefetches, and from
// how many CTAs: all of it, up to half of L2, when x takes at most three
// quarters of L2; nothing when it does not (at T = 32768 x is 470 MB and a
// partial prefetch measured slower).  Alternating A/B, three runs each:
// dsv3 149.3 -> 146.6 us per step, kimi 214.9 -> 213.3 us; prefill and
// mixtral unchanged.
void prefetch_plan(int64_t x_bytes, int64_t &pf_bytes, int &pf_ctas)
{
    struct Dev {
        std::atomic<int64_t> l2{-1};
        std::atomic<int> nsm{0};
    };
    static Dev devs[64];
    pf_bytes = 0;
    pf_ctas = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return;
    Dev &d = devs[dev];
    int64_t l2 = d.l2.load(std::memory_order_relaxed);
    int nsm = d.nsm.load(std::memory_order_relaxed);
    if (l2 < 0) {
        int v = 0, m = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrL2CacheSize, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&m, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return;
        }
        l2 = v;
        nsm = m;
        d.nsm.store(nsm, std::memory_order_relaxed);
        d.l2.store(l2, std::memory_order_relaxed);
    }
    if (x_bytes <= 0 || nsm < 1 || x_bytes > 3 * l2 / 4)
        return;
    pf_bytes = std::min<int64_t>(x_bytes, l2 / 2) / 16 * 16;
    pf_ctas = 2 * nsm;  // about a first wave of CTAs
}

cudaError_t dispatch_bf16(const uint16_t *x, int T, int H, int k, const int32_t *dispatch_pos,
                          uint16_t *recv_x, int64_t rows, int32_t *dev_status, cudaStream_t s)
{
    const int nvec = H / 8;
    int64_t pf_bytes;
    int pf_ctas;
    prefetch_plan(static_cast<int64_t>(T) * H * 2, pf_bytes, pf_ctas);
    return launch_pdl(k_dispatch_bf16, dim3(T), dim3(threads_for(nvec)), 0, s,
                      reinterpret_cast<const uint4 *>(x), nvec, k, dispatch_pos,
                      reinterpret_cast<uint4 *>(recv_x), rows, dev_status, pf_bytes, pf_ctas);
}

cudaError_t dispatch_fp8(const uint16_t *x, int T, int H, int k, const int32_t *dispatch_pos,
                         uint8_t *recv_q, float *recv_scale, int64_t rows, int64_t scale_ld,
                         int32_t *dev_status, cudaStream_t s)
{
    int64_t pf_bytes;
    int pf_ctas;
    prefetch_plan(static_cast<int64_t>(T) * H * 2, pf_bytes, pf_ctas);
    if (pf_bytes == 0 && H % 256 == 0 && reinterpret_cast<uintptr_t>(recv_q) % 32 == 0)
        return launch_pdl(k_dispatch_fp8_w32, dim3(T), dim3(threads_for(H / 32)), 0, s,
                          reinterpret_cast<const uint4 *>(x), H, k, dispatch_pos, recv_q,
                          recv_scale, rows, scale_ld, dev_status);
    return launch_pdl(k_dispatch_fp8, dim3(T), dim3(threads_for(H / 16)), 0, s,
                      reinterpret_cast<const uint4 *>(x), H, k, dispatch_pos, recv_q, recv_scale,
                      rows, scale_ld, dev_status, pf_bytes, pf_ctas);
}

cudaError_t quantize_e4m3(const float *v, int64_t n, uint8_t *q, cudaStream_t s)
{
    const int64_t pairs = (n + 1) / 2;
    const int64_t blocks = (pairs + 255) / 256;
    const int grid = static_cast<int>(blocks < 148 * 32 ? blocks : 148 * 32);
    k_quantize_e4m3<<<grid, 256, 0, s>>>(v, n, q);
    return cudaGetLastError();
}

}  // namespace moe
