// compact.cu -- receiver side of the two-phase dispatch: copy every slot's
// row from its private (expert, source rank) region into the packed
// per-expert layout.
//
// "Efficient and portable mixture-of-experts communication", "Kernels
// portáteis": each rank keeps private storage to receive from every other
// rank, sized by the fixed number of tokens a source rank may send to each
// local expert, so senders write without synchronising; after receiving,
// the kernels reorganise the tokens into the layout the expert kernels
// need.  "Despacho": tokens are copied from that storage into contiguous
// buffers that become the inputs of the downstream kernels.
//
// On one GPU the sender's private rows and the receiver's packed rows are in
// the same memory; this copy is the extra pass the two-phase design pays
// compared with scattering straight into the packed rows.  One CTA per token
// copies its k rows with 16-byte loads that skip L1 and streaming stores.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kMaxK = 32;
constexpr int kMaxThreads = 512;

// Private and packed row of each of the token's slots, checked against the
// buffers; a slot with either row out of range is reported and skipped.
__device__ __forceinline__ void load_pairs(const int32_t *__restrict__ private_pos,
                                           const int32_t *__restrict__ dispatch_pos, int g, int k,
                                           int64_t private_rows, int64_t rows, int32_t *spr,
                                           int32_t *sdr, int32_t *dev_status)
{
    pdl_wait();
    if (threadIdx.x < k) {
        int pr = private_pos[static_cast<size_t>(g) * k + threadIdx.x];
        int dr = dispatch_pos[static_cast<size_t>(g) * k + threadIdx.x];
        if (pr < -1 || pr >= private_rows || dr < -1 || dr >= rows) {
            report(dev_status, MOE_ERR_INVALID_ARG);
            pr = dr = -1;
        }
        if (pr < 0 || dr < 0)
            pr = dr = -1;
        spr[threadIdx.x] = pr;
        sdr[threadIdx.x] = dr;
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kMaxThreads)
    k_compact_fp8(const uint4 *__restrict__ priv_q, const float *__restrict__ priv_scale,
                  int64_t private_rows, const int32_t *__restrict__ private_pos,
                  const int32_t *__restrict__ dispatch_pos, int H, int k, uint4 *__restrict__ recv_q,
                  float *__restrict__ recv_scale, int64_t rows, int32_t *__restrict__ dev_status)
{
    __shared__ int32_t spr[kMaxK], sdr[kMaxK];
    const int g = blockIdx.x;
    load_pairs(private_pos, dispatch_pos, g, k, private_rows, rows, spr, sdr, dev_status);
    const int nvec = H / 16;
    const int S = H / 128;
    for (int j = 0; j < k; ++j) {
        const int pr = spr[j], dr = sdr[j];
        if (pr < 0)
            continue;
        const uint4 *src = priv_q + static_cast<size_t>(pr) * nvec;
        uint4 *dst = recv_q + static_cast<size_t>(dr) * nvec;
        for (int v = threadIdx.x; v < nvec; v += blockDim.x)
            st_stream_v4(dst + v, ld_stream_v4(src + v));
        for (int b = threadIdx.x; b < S; b += blockDim.x)
            __stcs(recv_scale + static_cast<size_t>(dr) * S + b,
                   __ldg(priv_scale + static_cast<size_t>(pr) * S + b));
    }
    pdl_trigger();
}

__global__ void __launch_bounds__(kMaxThreads)
    k_compact_bf16(const uint4 *__restrict__ priv_x, int64_t private_rows,
                   const int32_t *__restrict__ private_pos, const int32_t *__restrict__ dispatch_pos,
                   int nvec, int k, uint4 *__restrict__ recv_x, int64_t rows,
                   int32_t *__restrict__ dev_status)
{
    __shared__ int32_t spr[kMaxK], sdr[kMaxK];
    const int g = blockIdx.x;
    load_pairs(private_pos, dispatch_pos, g, k, private_rows, rows, spr, sdr, dev_status);
    for (int j = 0; j < k; ++j) {
        const int pr = spr[j], dr = sdr[j];
        if (pr < 0)
            continue;
        const uint4 *src = priv_x + static_cast<size_t>(pr) * nvec;
        uint4 *dst = recv_x + static_cast<size_t>(dr) * nvec;
        for (int v = threadIdx.x; v < nvec; v += blockDim.x)
            st_stream_v4(dst + v, ld_stream_v4(src + v));
    }
    pdl_trigger();
}

int threads_for(int units)
{
    const int passes = ceil_div(units, kMaxThreads);
    return round_up(ceil_div(units, passes), 32);
}

}  // namespace

cudaError_t compact_fp8(const uint8_t *priv_q, const float *priv_scale, int64_t private_rows,
                        const int32_t *private_pos, const int32_t *dispatch_pos, int T, int H,
                        int k, uint8_t *recv_q, float *recv_scale, int64_t rows,
                        int32_t *dev_status, cudaStream_t s)
{
    return launch_pdl(k_compact_fp8, dim3(T), dim3(threads_for(H / 16)), 0, s,
                      reinterpret_cast<const uint4 *>(priv_q), priv_scale, private_rows,
                      private_pos, dispatch_pos, H, k, reinterpret_cast<uint4 *>(recv_q),
                      recv_scale, rows, dev_status);
}

cudaError_t compact_bf16(const uint16_t *priv_x, int64_t private_rows, const int32_t *private_pos,
                         const int32_t *dispatch_pos, int T, int H, int k, uint16_t *recv_x,
                         int64_t rows, int32_t *dev_status, cudaStream_t s)
{
    const int nvec = H / 8;
    return launch_pdl(k_compact_bf16, dim3(T), dim3(threads_for(nvec)), 0, s,
                      reinterpret_cast<const uint4 *>(priv_x), private_rows, private_pos,
                      dispatch_pos, nvec, k, reinterpret_cast<uint4 *>(recv_x), rows, dev_status);
}

}  // namespace moe
