// search_noalloc.cu -- awq_scale_search_noalloc: the fused alpha-grid scale
// search for callers that cannot allocate device memory.
//
// Some callers have no way to obtain scratch memory: a plug-in whose host
// framework owns every device allocation through its own arena and exposes no
// allocator to plug-ins, a latency-critical section where a cudaMalloc (which
// may synchronise the device) is not acceptable, or a plain C caller that only
// holds pointers to its own inputs and outputs.  For them this entry point
// takes the same inputs and outputs as awq_scale_search but no workspace: its
// scratch is the file-scope array below, kNoAllocScratchBytes per device.
//
// Properties a caller must know:
//   * the array is a static device symbol, so every GPU on which this library
//     is used holds kNoAllocScratchBytes of it until the process exits;
//   * the first call on a device looks up the array's device address with
//     cudaGetSymbolAddress (with that device current) and caches it for the
//     life of the process; make that first call before any stream capture on
//     that device.  A cudaDeviceReset destroys the context the address
//     belongs to, so the cached address is stale afterwards: do not call this
//     entry point on a device after resetting it;
//   * every call on a device shares the one array and it keeps the previous
//     call's contents.  The kernels overwrite every scratch byte they read
//     (scale tables, per-CTA partial sums) and clear the error word first, so
//     a call never depends on old contents -- but two calls that overlap on
//     the GPU (different streams, no ordering between them) race on it;
//   * sizes whose scratch need exceeds kNoAllocScratchBytes are rejected with
//     AWQ_ERR_WORKSPACE before anything is enqueued;
//   * nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = AWQ_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_search_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_search_scratch on the current device (looked up once
// per device; the host-side name of the array is not a device address).
awq_status scratch_on_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return AWQ_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return AWQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_search_scratch) != cudaSuccess || !p)
            return AWQ_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return AWQ_OK;
}

}  // namespace

extern "C" awq_status awq_scale_search_noalloc(int n_seg, const void* const* W,
                                               const int64_t* d_out, int64_t d_in,
                                               const float* x_mean, int group_size,
                                               int n_grid, int flags, double* err,
                                               int32_t* best_idx, float* s_best,
                                               void* stream) {
    // Argument checks first, through the workspace entry point itself with no
    // workspace: it validates every argument and then, finding no workspace,
    // returns AWQ_ERR_WORKSPACE with nothing enqueued.  Any other code is an
    // argument error, reported exactly as awq_scale_search reports it.
    const awq_status pre = awq_scale_search(n_seg, W, d_out, d_in, x_mean, group_size,
                                            n_grid, flags, err, best_idx, s_best, nullptr, 0,
                                            stream);
    if (pre != AWQ_ERR_WORKSPACE) return pre;
    void* scratch = nullptr;
    const awq_status s2 = scratch_on_current_device(&scratch);
    if (s2 != AWQ_OK) return s2;
    // a size whose workspace need exceeds the array is rejected there with
    // AWQ_ERR_WORKSPACE, again before anything is enqueued
    return awq_scale_search(n_seg, W, d_out, d_in, x_mean, group_size, n_grid, flags, err,
                            best_idx, s_best, scratch, kNoAllocScratchBytes, stream);
}
