// tc_prefill_no_alloc: tc_prefill for callers that cannot allocate device
// memory.
//
// Some callers have no way to obtain scratch space: code running inside a
// framework that owns every allocation and forbids cudaMalloc during a step,
// real-time paths where an allocation may block or fail, and plugins loaded
// into a host process that exposes no allocator.  For them this entry point
// uses a fixed scratch array compiled into the library instead of a caller
// workspace.  The array is a file-scope __device__ variable, so every GPU
// that loads the library holds TC_NO_ALLOC_SCRATCH_BYTES of it until the
// process exits.
//
// Its device address is looked up once per device with cudaGetSymbolAddress
// (a host-side use of the array's name is not a device address) on the first
// call made while that device is current; that first call should therefore
// happen before any stream capture.  The address is cached for the life of
// the context: after cudaDeviceReset the array may move, so the cache entry
// is dropped when a call fails with a CUDA error, and callers should not rely
// on the entry point across a device reset without making a fresh first call.
// All calls share the one array: its
// contents are whatever the previous call left there, which is harmless
// because the prefill writes every scratch byte before reading it, and two
// calls whose kernels overlap on the GPU (different streams, no ordering
// between them) race on it.  Nothing here calls cudaMalloc, cudaFree or any
// allocating library routine.

#include <cuda_runtime.h>

#include <mutex>

#include "tc.h"
#include "tc_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_scratch[TC_NO_ALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device (nullptr on failure).
void *scratch_address(int dev) {
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_scratch_ptr[dev] = ptr;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" tc_status tc_prefill_no_alloc(const tc_prefill_desc *desc, const void *q,
                                         const void *k, const void *v, const float *lambda,
                                         const float *eta, const float *g, void *y,
                                         float *A_final, tc_stream_t stream) {
    size_t need = tc_prefill_workspace_size(desc);
    if (need == (size_t)-1) return TC_ERR_INVALID_ARG;
    // Under TC_PATH_AUTO a call whose general-path scratch (per-chunk states)
    // does not fit runs on the fused kernel when that one's does.
    int path = -1;
    if (need > (size_t)TC_NO_ALLOC_SCRATCH_BYTES && tc_get_prefill_path() == TC_PATH_AUTO) {
        tc::ScopedPrefillPath fused(TC_PATH_FUSED);
        const size_t f = tc_prefill_workspace_size(desc);
        if (f <= (size_t)TC_NO_ALLOC_SCRATCH_BYTES) {
            need = f;
            path = TC_PATH_FUSED;
        }
    }
    if (need > (size_t)TC_NO_ALLOC_SCRATCH_BYTES) return TC_ERR_WORKSPACE;
    tc::ScopedPrefillPath chosen(path);
    int count = 0, dev = 0;
    if (cudaGetDeviceCount(&count) != cudaSuccess || count == 0 || cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return TC_ERR_NO_DEVICE;
    }
    void *scratch = scratch_address(dev);
    if (!scratch) return TC_ERR_CUDA;
    const tc_status st = tc_prefill(desc, q, k, v, lambda, eta, g, y, A_final, scratch,
                                    (size_t)TC_NO_ALLOC_SCRATCH_BYTES, stream);
    if (st == TC_ERR_CUDA) {
        // the cached address may belong to a context that no longer exists
        // (cudaDeviceReset): look it up again on the next call
        std::lock_guard<std::mutex> lock(g_mutex);
        g_scratch_ptr[dev] = nullptr;
    }
    return st;
}
