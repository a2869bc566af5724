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
// device address is obtained with cudaGetSymbolAddress, with the device
// current (set up by the first call on each device, refreshed by every call
// made outside stream capture), and passed to the kernels like any workspace.
#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "kernels.cuh"
#include "moe_route.h"

namespace {

__device__ __align__(256) int32_t g_layout_scratch[MOE_LAYOUT_NOALLOC_SCRATCH_BYTES / sizeof(int32_t)];

std::mutex g_setup_mutex;
std::vector<void *> g_scratch_ptr;  // per device ordinal, sized from cudaGetDeviceCount

// Device address of g_layout_scratch on the current device.  Outside stream
// capture it is looked up again on every call (cudaGetSymbolAddress is a host
// query and allocates nothing), so a context that was torn down and created
// again (cudaDeviceReset, a released and re-retained primary context) never
// sees a stale address.  While `stream` is capturing, the address kept by the
// last call outside capture is used: the first call on a device must come
// before any capture on it, else MOE_ERR_UNSUPPORTED.
int scratch_on_current_device(cudaStream_t stream, void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0)
        return MOE_ERR_CUDA;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    bool capturing = true;  // when the query itself fails, do not risk a lookup
    if (cudaStreamIsCapturing(stream, &cs) == cudaSuccess)
        capturing = (cs != cudaStreamCaptureStatusNone);
    else
        cudaGetLastError();
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (static_cast<size_t>(dev) >= g_scratch_ptr.size()) {
        int n = 0;
        if (cudaGetDeviceCount(&n) != cudaSuccess || n <= dev)
            return MOE_ERR_CUDA;
        g_scratch_ptr.resize(static_cast<size_t>(n), nullptr);
    }
    if (!capturing) {
        void *p = nullptr;
        const cudaError_t err = cudaGetSymbolAddress(&p, g_layout_scratch);
        if (err != cudaSuccess || p == nullptr)
            return MOE_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    } else if (g_scratch_ptr[dev] == nullptr) {
        return MOE_ERR_UNSUPPORTED;  // never set up on this device outside a capture
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
        const int st = scratch_on_current_device(static_cast<cudaStream_t>(stream), &scratch);
        if (st != MOE_OK)
            return st;
    }
    return moe_dispatch_layout(topk_idx, T, k, E, R, capacity, rows, expert_counts,
                               expert_src_counts, rank_counts, expert_offsets, dispatch_pos,
                               recv_src, scratch, MOE_LAYOUT_NOALLOC_SCRATCH_BYTES, dev_status,
                               stream);
}
