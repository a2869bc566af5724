// combine.cu -- gather each token's k expert rows and form the router-
// weighted sum in fp32, stored as bf16.
//
// "Efficient and portable mixture-of-experts communication", "Combinação":
// the receiver reads the routing table to know which buffer to read and which
// weight each expert contribution gets, and computes their weighted sum;
// "Enabling trillion-parameter models on AWS EFA", "Dağıtım/Birleştirme
// Gecikmesi": bf16 combine, accumulation only at the receiver.
//
// One CTA per token; a thread owns 8 consecutive channels (16 bytes of each
// row).  The token's row indices and weights are held in registers, so all
// k (up to 8) 16-byte loads of a pass issue back to back before any is used;
// then the sum runs in ascending j with a separate binary32 multiply and add
// per term (__fmul_rn / __fadd_rn are never contracted into an FMA), so the
// output is bit-reproducible.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kMaxK = 32;
constexpr int kMaxThreads = 512;

// KREG rows and weights live in registers (read from shared memory once, after
// the CTA has validated them), so the loads of a pass need no shared-memory
// round trip; terms beyond KREG (k > 8) follow in order from shared memory.
template <int KREG>
__global__ void __launch_bounds__(kMaxThreads)
    k_combine_bf16(const uint4 *__restrict__ y, const int32_t *__restrict__ dispatch_pos,
                   const float *__restrict__ topk_w, int nvec, int k, int64_t rows,
                   uint4 *__restrict__ out, int32_t *__restrict__ dev_status)
{
    __shared__ int32_t srow[kMaxK];
    __shared__ float sw[kMaxK];
    const int g = blockIdx.x;
    pdl_wait();
    if (threadIdx.x < k) {
        int r = dispatch_pos[static_cast<size_t>(g) * k + threadIdx.x];
        if (r < -1 || r >= rows) {
            report(dev_status, MOE_ERR_INVALID_ARG);
            r = -1;
        }
        srow[threadIdx.x] = r;
        sw[threadIdx.x] = topk_w[static_cast<size_t>(g) * k + threadIdx.x];
    }
    __syncthreads();
    int rr[KREG];
    float ww[KREG];
#pragma unroll
    for (int j = 0; j < KREG; ++j) {
        rr[j] = (j < k) ? srow[j] : -1;
        ww[j] = (j < k) ? sw[j] : 0.0f;
    }

    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
        float acc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
            acc[c] = 0.0f;
        uint4 d[KREG];
#pragma unroll
        for (int j = 0; j < KREG; ++j)
            d[j] = (rr[j] >= 0) ? ld_stream_v4(y + static_cast<size_t>(rr[j]) * nvec + v)
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
        // k > KREG: the remaining terms, in order, from shared memory
        for (int j = KREG; j < k; ++j) {
            const int r = srow[j];
            if (r < 0)
                continue;
            const uint4 e = ld_stream_v4(y + static_cast<size_t>(r) * nvec + v);
            const uint32_t wds[4] = {e.x, e.y, e.z, e.w};
            const float wj = sw[j];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(wj, bf16_lo(wds[i])));
                acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __fmul_rn(wj, bf16_hi(wds[i])));
            }
        }
        const uint4 o = make_uint4(bf16x2_rn(acc[0], acc[1]), bf16x2_rn(acc[2], acc[3]),
                                   bf16x2_rn(acc[4], acc[5]), bf16x2_rn(acc[6], acc[7]));
        st_stream_v4(out + static_cast<size_t>(g) * nvec + v, o);
    }
    pdl_trigger();
}

int threads_for(int units)
{
    const int passes = ceil_div(units, kMaxThreads);
    return round_up(ceil_div(units, passes), 32);
}

}  // namespace

cudaError_t combine_bf16(const uint16_t *y, const int32_t *dispatch_pos, const float *topk_w,
                         int T, int H, int k, int64_t rows, uint16_t *out, int32_t *dev_status,
                         cudaStream_t s)
{
    const int nvec = H / 8;
    const dim3 grid(T), block(threads_for(nvec));
    const uint4 *yv = reinterpret_cast<const uint4 *>(y);
    uint4 *ov = reinterpret_cast<uint4 *>(out);
    if (k <= 2)
        return launch_pdl(k_combine_bf16<2>, grid, block, 0, s, yv, dispatch_pos, topk_w, nvec, k,
                          rows, ov, dev_status);
    if (k <= 4)
        return launch_pdl(k_combine_bf16<4>, grid, block, 0, s, yv, dispatch_pos, topk_w, nvec, k,
                          rows, ov, dev_status);
    return launch_pdl(k_combine_bf16<8>, grid, block, 0, s, yv, dispatch_pos, topk_w, nvec, k, rows,
                      ov, dev_status);
}

}  // namespace moe
