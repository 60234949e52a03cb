// chunk_common.cuh -- pieces shared by the tensor-core chunk kernels: chunk length, swizzled
// tile stores (including bf16 hi/lo pairs), TMEM row loads, the split-precision MMA helper and the
// blocked unit-lower-triangular inverse.
#pragma once

#include "tc.cuh"

namespace prism {
namespace {

using namespace tc;

constexpr int C = 64;         // chunk length of the tensor-core path
constexpr int AS = C + 1;     // padded fp32 row stride of the solve matrix

__device__ __forceinline__ void st16(uint8_t *base, uint32_t off, uint4 v) {
    *reinterpret_cast<uint4 *>(base + off) = v;
}

template <int BV>
__device__ __forceinline__ uint32_t vt_off(int row, int col) {
    // x BV tile: 64B swizzle when BV = 32, 128B when BV = 64
    if constexpr (BV == 32) return sw64_off(row, col);
    else return sw128_off(row, col, 0);
}

template <int BV>
__device__ __forceinline__ uint64_t desc_vt(uint32_t base, int ks) {
    if constexpr (BV == 32) return desc_mn_sw64(base, ks);
    else return desc_mn_sw128(base, ks, C * 128);  // a single MN block; LBO unused
}

// hi / lo bf16 pair of 8 floats
__device__ __forceinline__ void split8(const float *x, uint4 &hi, uint4 &lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 hh = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
        float2 hf = __bfloat1622float2(hh);
        __nv_bfloat162 ll = __floats2bfloat162_rn(x[2 * i] - hf.x, x[2 * i + 1] - hf.y);
        h[i] = *reinterpret_cast<uint32_t *>(&hh);
        l[i] = *reinterpret_cast<uint32_t *>(&ll);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// A row of BV fp32 values as a hi / lo pair into two x BV tiles.
template <int BV>
__device__ __forceinline__ void store_row_split(uint8_t *hi, uint8_t *lo, int row, const float *x) {
#pragma unroll
    for (int c8 = 0; c8 < BV / 8; ++c8) {
        uint4 h, l;
        split8(x + c8 * 8, h, l);
        const uint32_t off = vt_off<BV>(row, c8 * 8);
        st16(hi, off, h);
        st16(lo, off, l);
    }
}

// 32 fp32 values at (row, col .. col+31) of K-major SW128 tiles, as a hi / lo pair or hi only.
__device__ __forceinline__ void store32_split(uint8_t *hi, uint8_t *lo, int row, int col,
                                              const float *x, uint32_t block_bytes = 0) {
#pragma unroll
    for (int c8 = 0; c8 < 4; ++c8) {
        uint4 h, l;
        split8(x + c8 * 8, h, l);
        const uint32_t off = sw128_off(row, col + c8 * 8, block_bytes);
        st16(hi, off, h);
        if (lo) st16(lo, off, l);
    }
}

// BV consecutive TMEM columns of this thread's lane (warp-collective).
template <int BV>
__device__ __forceinline__ void ld_row(uint32_t tbase, int warp, uint32_t col, float *x) {
#pragma unroll
    for (int c = 0; c < BV; c += 32) {
        float v[32];
        tmem_ld32(taddr(tbase, 32 * warp, col + c), v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) x[c + j] = v[j];
    }
}

// Shared-memory writes become visible to the tensor core and earlier tcgen05.ld complete before
// the issuing thread proceeds.
__device__ __forceinline__ void sync_for_mma() {
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
}

// D (+)= (A_hi + A_lo)(B_hi + B_lo) without the lo*lo term; K = 16 * nks.  Pass alo / blo = 0 to
// skip a split.  `acc` says whether the first product accumulates onto D.
template <class FA, class FB>
__device__ __forceinline__ void mma_split(uint32_t d, uint32_t idesc, int nks, FA adesc, FB bdesc,
                                          uint32_t ahi, uint32_t alo, uint32_t bhi, uint32_t blo,
                                          bool acc) {
    for (int ks = 0; ks < nks; ++ks) mma_bf16(d, adesc(ahi, ks), bdesc(bhi, ks), idesc, acc || ks > 0);
    if (blo)
        for (int ks = 0; ks < nks; ++ks) mma_bf16(d, adesc(ahi, ks), bdesc(blo, ks), idesc, 1);
    if (alo)
        for (int ks = 0; ks < nks; ++ks) mma_bf16(d, adesc(alo, ks), bdesc(bhi, ks), idesc, 1);
}

// T = (I + A)^{-1} for strictly lower-triangular A (C = 64), blocked: the four 16 x 16 diagonal
// blocks by forward substitution, then two doubling levels T_21 = -T_22 A_21 T_11 (16 -> 32 -> 64)
// as register-blocked products with fixed trip counts.  Safe in place (A == Tm): every block is
// read as A before it is overwritten with T.  Run by 128 threads (tid < 128); SYNC(), a barrier
// among exactly those threads, separates its phases.  tmp holds 32 x 33 floats.
struct CtaSync {
    __device__ __forceinline__ void operator()() const { __syncthreads(); }
};

template <int NTH, class SYNC = CtaSync>
__device__ void solve_unit_lower(const float *A, float *Tm, float *tmp, int tid, SYNC sync = SYNC()) {
    static_assert(NTH == 128, "the solve is laid out for 128 threads");
    const int warp = tid >> 5, lane = tid & 31;
    // diagonal blocks: warp w inverts block w, lane j < 16 computes column j
    if (lane < 16) {
        const int o = 16 * warp, j = lane;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float s = (i == j) ? 1.f : 0.f;
#pragma unroll
            for (int k = 0; k < i; ++k) s = fmaf(-A[(o + i) * AS + o + k], x[k], s);
            x[i] = (i < j) ? 0.f : s;
        }
        __syncwarp(0x0000ffffu);  // every lane has read the block before any lane overwrites it
#pragma unroll
        for (int i = 0; i < 16; ++i) Tm[(o + i) * AS + o + j] = x[i];
    }
    sync();
    // level 1, 16-blocks, pairs p = 0, 1: rows r0 = 32p + 16, cols c0 = 32p; thread: 1 row x 4 cols
    {
        const int pp = tid >> 6, r = (tid >> 2) & 15, cq = (tid & 3) * 4;
        const int r0 = 32 * pp + 16, c0 = 32 * pp;
        float m[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float a = A[(r0 + r) * AS + c0 + k];
#pragma unroll
            for (int j = 0; j < 4; ++j) m[j] = fmaf(a, Tm[(c0 + k) * AS + c0 + cq + j], m[j]);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) tmp[pp * 16 * 17 + r * 17 + cq + j] = m[j];
        sync();
#pragma unroll
        for (int j = 0; j < 4; ++j) m[j] = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float t = Tm[(r0 + r) * AS + r0 + k];
#pragma unroll
            for (int j = 0; j < 4; ++j) m[j] = fmaf(t, tmp[pp * 16 * 17 + k * 17 + cq + j], m[j]);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) Tm[(r0 + r) * AS + c0 + cq + j] = -m[j];
    }
    sync();
    // level 2, 32-blocks: rows 32.., cols 0..31; thread: 1 row x 8 cols
    {
        const int r = tid >> 2, cq = (tid & 3) * 8;
        float m[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) m[j] = 0.f;
#pragma unroll 8
        for (int k = 0; k < 32; ++k) {
            const float a = A[(32 + r) * AS + k];
#pragma unroll
            for (int j = 0; j < 8; ++j) m[j] = fmaf(a, Tm[k * AS + cq + j], m[j]);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) tmp[r * 33 + cq + j] = m[j];
        sync();
#pragma unroll
        for (int j = 0; j < 8; ++j) m[j] = 0.f;
#pragma unroll 8
        for (int k = 0; k < 32; ++k) {
            const float t = Tm[(32 + r) * AS + 32 + k];
#pragma unroll
            for (int j = 0; j < 8; ++j) m[j] = fmaf(t, tmp[k * 33 + cq + j], m[j]);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) Tm[(32 + r) * AS + cq + j] = -m[j];
    }
    sync();
}

}  // namespace
}  // namespace prism
