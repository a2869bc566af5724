// layout_noalloc.cu -- moe_dispatch_layout_noalloc: the layout entry point
// for callers that cannot allocate device memory.
//
// moe_dispatch_layout needs a caller-supplied workspace (per-chunk
// histograms).  Some callers cannot provide one: code that runs where
// cudaMalloc is not allowed or not wanted -- a plugin or custom-op layer that
// is handed only input and output buffers and no allocator, a host callback
// or a latency-critical loop where cudaMalloc would synchronise the device,
// or a deployment whose device memory budget is fixed up front.  This entry
// point takes the same inputs and outputs but no workspace: it uses a
// file-scope device array of fixed size instead, and it allocates nothing.
//
// The array is one static __device__ object of this library, so every GPU
// that loads the library holds its 1 MiB until the process exits.  In host
// code its name is only a host-side stand-in, never a device address; the
// device address is obtained once per device with cudaGetSymbolAddress,
// with that device current, and passed to the kernels like any workspace.
#include <cuda_runtime.h>

#include <mutex>

#include "kernels.cuh"
#include "moe_route.h"

namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) int32_t g_layout_scratch[MOE_LAYOUT_NOALLOC_SCRATCH_BYTES / sizeof(int32_t)];

std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_layout_scratch on the current device (set up on the
// first call for that device).
int scratch_on_current_device(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        const cudaError_t err = cudaGetSymbolAddress(&p, g_layout_scratch);
        if (err != cudaSuccess || p == nullptr)
            return MOE_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" int moe_dispatch_layout_noalloc(const int32_t *topk_idx, int T, int k, int E, int R,
                                           int capacity, int64_t rows, int32_t *expert_counts,
                                           int32_t *expert_src_counts, int32_t *rank_counts,
                                           int32_t *expert_offsets, int32_t *dispatch_pos,
                                           int32_t *recv_src, int32_t *dev_status, void *stream)
{
    const size_t need = moe_layout_workspace_bytes(T, k, E, R);
    if (need > MOE_LAYOUT_NOALLOC_SCRATCH_BYTES)
        return MOE_ERR_WORKSPACE;  // this (T, k, E, R) needs more than the fixed scratch
    void *scratch = nullptr;
    if (need > 0) {  // need == 0: invalid sizes, rejected below before any launch
        const int st = scratch_on_current_device(&scratch);
        if (st != MOE_OK)
            return st;
    }
    return moe_dispatch_layout(topk_idx, T, k, E, R, capacity, rows, expert_counts,
                               expert_src_counts, rank_counts, expert_offsets, dispatch_pos,
                               recv_src, scratch, MOE_LAYOUT_NOALLOC_SCRATCH_BYTES, dev_status,
                               stream);
}
