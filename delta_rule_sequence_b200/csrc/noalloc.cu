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
// host-side handle, so its device address is looked up with cudaGetSymbolAddress, with the device
// current, on the first call on each device (and again if that device's context has changed, for
// example after a cudaDeviceReset), and cached.  Its first 4 bytes are the scan's status word:
// zero at load, written only by a kernel whose bounded wait gave up, and read and cleared by
// prism_query_device_status.  Nothing else in it has to start at zero.

#include <mutex>

#include <cuda.h>

#include "common.cuh"

namespace prism {
prism_status check_scan_call(const prism_shape *shape, const void *q, const void *k, const void *v,
                             const float *alpha, const float *beta, const void *u, const void *w,
                             const float *S0, const void *o, const float *S_final);
}  // namespace prism

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[PRISM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
struct ScratchSlot {
    void *ctx = nullptr;   // the context the address was looked up in
    void *addr = nullptr;  // device address of g_noalloc_scratch in that context
};
ScratchSlot g_slots[kMaxDevices];
std::mutex g_scratch_mutex;

// The driver's cuCtxGetCurrent, fetched once through the runtime (no libcuda link).
using CtxGetCurrent = CUresult (*)(CUcontext *);
CtxGetCurrent ctx_get_current() {
    static CtxGetCurrent fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrent>(ptr);
    });
    return fn;
}

// Device address of the scratch array on the current device.
prism_status scratch_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return PRISM_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return PRISM_ERR_UNSUPPORTED;
    CtxGetCurrent get = ctx_get_current();
    if (!get) return PRISM_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (get(&ctx) != CUDA_SUCCESS) return PRISM_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    ScratchSlot &slot = g_slots[dev];
    if (slot.addr == nullptr || ctx == nullptr || slot.ctx != (void *)ctx) {
        // the lookup also makes the device's primary context current if no context was
        void *addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || addr == nullptr)
            return PRISM_ERR_CUDA;
        if (get(&ctx) != CUDA_SUCCESS || ctx == nullptr) return PRISM_ERR_CUDA;
        slot.ctx = (void *)ctx;
        slot.addr = addr;
    }
    *out = slot.addr;
    return PRISM_OK;
}

}  // namespace

namespace prism {
// Read and clear the status word at the start of the current device's scratch.
cudaError_t noalloc_status(uint32_t *out) {
    uint32_t word = 0;
    cudaError_t err = cudaMemcpyFromSymbol(&word, g_noalloc_scratch, sizeof word);
    if (err != cudaSuccess) return err;
    if (word != 0) {
        const uint32_t zero = 0;
        if ((err = cudaMemcpyToSymbol(g_noalloc_scratch, &zero, sizeof zero)) != cudaSuccess) return err;
    }
    *out = word;
    return cudaSuccess;
}
}  // namespace prism

extern "C" prism_status prism_scan_fwd_noalloc(const prism_shape *shape, const void *q,
                                               const void *k, const void *v, const float *alpha,
                                               const float *beta, const void *u, const void *w,
                                               const float *S0, void *o, float *S_final,
                                               void *stream) {
    // the same argument checks as prism_scan_fwd, and the same codes, before anything is sized
    prism_status st = prism::check_scan_call(shape, q, k, v, alpha, beta, u, w, S0, o, S_final);
    if (st != PRISM_OK) return st;
    size_t need = 0;
    st = prism_scan_fwd_workspace_size(shape, &need);
    if (st != PRISM_OK) return st;
    if (need > (size_t)PRISM_NOALLOC_SCRATCH_BYTES) return PRISM_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    st = scratch_address(&scratch);
    if (st != PRISM_OK) return st;
    return prism_scan_fwd(shape, q, k, v, alpha, beta, u, w, S0, o, S_final, scratch,
                          (size_t)PRISM_NOALLOC_SCRATCH_BYTES, stream);
}
