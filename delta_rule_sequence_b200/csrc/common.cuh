// common.cuh -- device helpers shared by the libprism kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/prism.h"

namespace prism {

// Arguments of one prism_scan_fwd call, as the kernels see them.
struct ScanArgs {
    int B, H, T, dk, dv, L, chunk;
    const void *q, *k, *v;
    const float *alpha, *beta;
    const void *u, *w;
    const float *S0;
    void *o;
    float *S_final;
    uint32_t *status;  // device status word (PRISM_OK / PRISM_ERR_TIMEOUT), may be null
    int flags;         // kNoWrite | kS0Identity | kNoOutput (segment passes of the segmented scan)
};

// Flags of a scan pass.  kNoWrite: the write term is zero (u = 0 / v = 0);  kS0Identity: the entry
// state's row r is the unit vector e_r (requires dk == dv), so S_final returns the pass's affine
// map E;  kNoOutput: o is not written;  kStallTest: the Gated-DeltaNet state kernel's load warp
// issues nothing and every wait gives up after a short limit (a test of the give-up path);
// kForceWkLo: the state kernel adds the Wk_lo term from the first chunk, whatever the state's size;
// kStallPrep, kStallDecode: the same give-up test for the per-chunk prep kernels (their tile loads
// are not issued) and for the bulk-copy decode kernel (its state copies are not issued).
enum : int { kNoWrite = 1, kS0Identity = 2, kNoOutput = 4, kStallTest = 8, kForceWkLo = 16,
             kStallPrep = 32, kStallDecode = 64 };

// Poll limits of the bounded mbarrier waits: normal operation, and the stall test.
constexpr uint32_t kWaitPolls = 1u << 24;
constexpr uint32_t kStallTestPolls = 1u << 12;

// Workspace layout: [0, 256) status block; segment data of the segmented scan after it.
constexpr size_t kStatusBytes = 256;

template <typename IO>
__device__ __forceinline__ float ld_io(const IO *p, size_t i);
template <>
__device__ __forceinline__ float ld_io<float>(const float *p, size_t i) { return p[i]; }
template <>
__device__ __forceinline__ float ld_io<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}

template <typename IO>
__device__ __forceinline__ void st_io(IO *p, size_t i, float x);
template <>
__device__ __forceinline__ void st_io<float>(float *p, size_t i, float x) { p[i] = x; }
template <>
__device__ __forceinline__ void st_io<__nv_bfloat16>(__nv_bfloat16 *p, size_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ float warp_inclusive_scan(float x, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

// Launch probe (prism_debug_record_launch_events): records the caller's next event on the stream
// right before a kernel launch of an armed call.  Every launcher calls it before each launch.
void launch_probe_mark(cudaStream_t s);

// Record a device-side failure without trapping: the first failure wins.
__device__ __forceinline__ void record_status(uint32_t *status, uint32_t code) {
    if (status) atomicCAS(status, (uint32_t)PRISM_OK, code);
}

}  // namespace prism
