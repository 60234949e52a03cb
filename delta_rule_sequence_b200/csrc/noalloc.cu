// noalloc.cu -- prism_scan_fwd for callers that cannot allocate device memory.
//
// Some callers have no way to obtain device scratch at the moment they run the scan: plugins
// inside an inference engine that owns every device allocation and forbids allocating while it
// executes, and latency-critical paths where cudaMalloc's implicit device-wide synchronisation is
// not acceptable.  For them this file owns a fixed scratch array in device global memory and runs
// the ordinary scan with it as the workspace.  The caller passes only inputs and outputs.
//
// The array is a file-scope __device__ object: every GPU that loads libprism.so holds
// PRISM_NOALLOC_SCRATCH_BYTES of it until the process exits.  In host code its name is only a
// host-side handle, so the device address is looked up once per device with
// cudaGetSymbolAddress (with that device current) and cached.

#include <mutex>

#include "common.cuh"

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[PRISM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device (looked up on first use).
prism_status scratch_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return PRISM_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return PRISM_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || addr == nullptr)
            return PRISM_ERR_CUDA;
        g_scratch_addr[dev] = addr;
    }
    *out = g_scratch_addr[dev];
    return PRISM_OK;
}

}  // namespace

extern "C" prism_status prism_scan_fwd_noalloc(const prism_shape *shape, const void *q,
                                               const void *k, const void *v, const float *alpha,
                                               const float *beta, const void *u, const void *w,
                                               const float *S0, void *o, float *S_final,
                                               void *stream) {
    if (!shape) return PRISM_ERR_INVALID_ARG;
    size_t need = 0;
    prism_status st = prism_scan_fwd_workspace_size(shape, &need);
    if (st != PRISM_OK) return st;
    if (need > (size_t)PRISM_NOALLOC_SCRATCH_BYTES) return PRISM_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    st = scratch_address(&scratch);
    if (st != PRISM_OK) return st;
    // No part of the scratch has to start at zero: the kernels only ever write its status word
    // (on a bounded-wait failure) and never read it back.
    return prism_scan_fwd(shape, q, k, v, alpha, beta, u, w, S0, o, S_final, scratch,
                          (size_t)PRISM_NOALLOC_SCRATCH_BYTES, stream);
}
