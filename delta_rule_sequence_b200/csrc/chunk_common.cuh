// chunk_common.cuh -- pieces shared by the tensor-core chunk kernels: chunk length, swizzled
// tile stores (including bf16 hi/lo pairs), TMEM row loads, the split-precision MMA helper and the
// blocked unit-lower-triangular inverse.
#pragma once

#include "tc.cuh"

namespace prism {
namespace {

using namespace tc;

constexpr int C = 64;         // chunk length of the tensor-core path
// fp32 row stride of the solve matrix: rows stay 16-byte aligned for vector loads, and the 4-word
// pad spreads eight consecutive rows over the eight 16-byte bank groups
constexpr int AS = C + 4;
constexpr int kTmp1 = 20, kTmp2 = 36;         // row strides of the solve's two product buffers
constexpr int kSolveTmpFloats = 32 * kTmp2;   // its scratch (the 16-block pair buffer fits inside)

// N consecutive fp32 in shared memory (16-byte aligned; 8-byte for N = 2) to / from registers
template <int N>
__device__ __forceinline__ void vld(const float *p, float *v) {
    if constexpr (N == 2) {
        const float2 a = *reinterpret_cast<const float2 *>(p);
        v[0] = a.x;
        v[1] = a.y;
    } else {
#pragma unroll
        for (int m = 0; m < N / 4; ++m) {
            const float4 a = reinterpret_cast<const float4 *>(p)[m];
            v[4 * m] = a.x;
            v[4 * m + 1] = a.y;
            v[4 * m + 2] = a.z;
            v[4 * m + 3] = a.w;
        }
    }
}
template <int N>
__device__ __forceinline__ void vst(float *p, const float *v) {
    if constexpr (N == 2) {
        *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
    } else {
#pragma unroll
        for (int m = 0; m < N / 4; ++m)
            reinterpret_cast<float4 *>(p)[m] = make_float4(v[4 * m], v[4 * m + 1], v[4 * m + 2], v[4 * m + 3]);
    }
}

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

// Two fp32 lanes per instruction (the packed f32x2 arithmetic of sm_100): d = a * b + c, each
// lane rounded as fmaf rounds it
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    unsigned long long ra, rb, rc, rd;
    asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(rc) : "f"(c.x), "f"(c.y));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
    float2 d;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
    return d;
}

// m[0..N) += a * v[0..N) for even N, two lanes an instruction
template <int N>
__device__ __forceinline__ void axpy2(float a, const float *v, float *m) {
    static_assert(N % 2 == 0, "pairs");
#pragma unroll
    for (int p = 0; p < N / 2; ++p) {
        const float2 r = ffma2(make_float2(a, a), make_float2(v[2 * p], v[2 * p + 1]), make_float2(m[2 * p], m[2 * p + 1]));
        m[2 * p] = r.x;
        m[2 * p + 1] = r.y;
    }
}

// T = (I + A)^{-1} for strictly lower-triangular A (C = 64), blocked: the four 16 x 16 diagonal
// blocks by forward substitution, then two doubling levels T_21 = -T_22 A_21 T_11 (16 -> 32 -> 64)
// as register-blocked products with fixed trip counts and vector shared-memory accesses.  Safe in
// place (A == Tm): every block is read as A before it is overwritten with T.  Run by NTH = 128 or
// 256 threads (tid < NTH); SYNC(), a barrier among exactly those threads, separates its phases.
// The diagonal blocks take warps 0-3; each doubling product spreads over all NTH threads (one
// row, 512 / NTH or 1024 / NTH columns a thread).  A, Tm and tmp are 16-byte aligned; tmp holds
// kSolveTmpFloats floats.
struct CtaSync {
    __device__ __forceinline__ void operator()() const { __syncthreads(); }
};

template <int NTH, class SYNC = CtaSync>
__device__ void solve_unit_lower(const float *A, float *Tm, float *tmp, int tid, SYNC sync = SYNC()) {
    static_assert(NTH == 128 || NTH == 256, "the solve is laid out for 128 or 256 threads");
    const int warp = tid >> 5, lane = tid & 31;
    // diagonal blocks: warp w < 4 inverts block w, lane j < 16 computes column j by forward
    // substitution in column order (once x_k is final it is eliminated from every later row, so
    // the dependent chain is 15 steps long, each step a set of independent FMAs)
    if (warp < 4 && lane < 16) {
        const int o = 16 * warp, j = lane;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = (i == j) ? 1.f : 0.f;
#pragma unroll
        for (int k = 0; k < 15; ++k) {
#pragma unroll
            for (int i = k + 1; i < 16; ++i) x[i] = fmaf(-A[(o + i) * AS + o + k], x[k], x[i]);
        }
        __syncwarp(0x0000ffffu);  // every lane has read the block before any lane overwrites it
#pragma unroll
        for (int i = 0; i < 16; ++i) Tm[(o + i) * AS + o + j] = x[i];
    }
    sync();
    constexpr int TPR = NTH / 32;  // threads per row of a doubling product
    // level 1, 16-blocks, pairs p = 0, 1: rows r0 = 32p + 16, cols c0 = 32p
    {
        constexpr int NC = 16 / TPR;
        const int pp = tid / (NTH / 2), r = (tid / TPR) & 15, cq = (tid % TPR) * NC;
        const int r0 = 32 * pp + 16, c0 = 32 * pp;
        float *tp = tmp + pp * 16 * kTmp1;
        float a[16], m[NC];
        vld<16>(A + (r0 + r) * AS + c0, a);  // row r of A_21
#pragma unroll
        for (int j = 0; j < NC; ++j) m[j] = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            float tv[NC];
            vld<NC>(Tm + (c0 + k) * AS + c0 + cq, tv);
            axpy2<NC>(a[k], tv, m);
        }
        vst<NC>(tp + r * kTmp1 + cq, m);
        sync();
        vld<16>(Tm + (r0 + r) * AS + r0, a);  // row r of T_22
#pragma unroll
        for (int j = 0; j < NC; ++j) m[j] = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            float tv[NC];
            vld<NC>(tp + k * kTmp1 + cq, tv);
            axpy2<NC>(a[k], tv, m);
        }
#pragma unroll
        for (int j = 0; j < NC; ++j) m[j] = -m[j];
        vst<NC>(Tm + (r0 + r) * AS + c0 + cq, m);
    }
    sync();
    // level 2, 32-blocks: rows 32.., cols 0..31; the 32-long rows are taken in two halves
    {
        constexpr int NC = 32 / TPR;
        const int r = tid / TPR, cq = (tid % TPR) * NC;
        float m[NC];
#pragma unroll
        for (int j = 0; j < NC; ++j) m[j] = 0.f;
#pragma unroll
        for (int kh = 0; kh < 2; ++kh) {
            float a[16];
            vld<16>(A + (32 + r) * AS + 16 * kh, a);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                float tv[NC];
                vld<NC>(Tm + (16 * kh + k) * AS + cq, tv);
                axpy2<NC>(a[k], tv, m);
            }
        }
        vst<NC>(tmp + r * kTmp2 + cq, m);
        sync();
#pragma unroll
        for (int j = 0; j < NC; ++j) m[j] = 0.f;
#pragma unroll
        for (int kh = 0; kh < 2; ++kh) {
            float a[16];
            vld<16>(Tm + (32 + r) * AS + 32 + 16 * kh, a);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                float tv[NC];
                vld<NC>(tmp + (16 * kh + k) * kTmp2 + cq, tv);
                axpy2<NC>(a[k], tv, m);
            }
        }
#pragma unroll
        for (int j = 0; j < NC; ++j) m[j] = -m[j];
        vst<NC>(Tm + (32 + r) * AS + cq, m);
    }
    sync();
}

}  // namespace
}  // namespace prism
