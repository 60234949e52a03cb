// producer.cu -- the input-anchored write-term producer in front of the scan: from each head's
// input sequence x and value v, the L write pairs (u_{t,l}, w_{t,l}) that prism_scan_fwd consumes.
//
// After "PRISM: Parallel Residual Iterative Sequence Model" (gist.science explainer), technical
// summary section 2.2 (input-anchored loop unrolling), the ShortConv width of the banbantang.com
// PRISM article, section 5(1) (the anchor sees the last 3-4 tokens) and its section 3(4) (the
// first residual is the input itself):
//   anchor      a_t = sum_{j=0..3} c_j * x_{t-j}                    (depthwise, causal)
//   directions  k^(l) = W_k^(l) a_t,  gains  p^(l) = W_p^(l) a_t       (every l at once)
//   residual    r^(1) = v_t,  delta^(l) = GELU(p^(l) * r^(l)),  r^(l+1) = r^(l) - delta^(l)
//   write       u_{t,l} = beta_t^(l) delta^(l),   w_{t,l} = k^(l)
// The anchor depends only on the input window, so every token's chain runs at once; the 2L
// projections of a token are one GEMM row against the stacked weights [W_k^(l); W_p^(l)].
//
// Both kernels work on tiles of 128 tokens of one (batch, head): epilogue warps build the anchor
// tile (the A operand, as a bf16 hi / lo pair: a single bf16 anchor lets the residual chain
// amplify its rounding past the bf16 output tolerance by the fourth rank) and hold the residual in
// registers (one token row a thread); one thread issues, for each l, one M = 128, N = 2d MMA of the
// anchor against the stacked weights into a TMEM accumulator, so the MMA of rank l + 1 runs while
// the epilogue of rank l reads k^(l) and p^(l), applies the GELU step and writes u and w.
//
// d = 64 (write_producer_ring_kernel): persistent, one CTA per SM walking a contiguous range of
// tiles (head-major, so a CTA's tiles share their weights).  A load warp brings each tile's x rows
// (with the 3-token causal halo; rows before the sequence start read as zeros) and v rows by TMA
// into swizzled shared memory while the previous tile is in its epilogue, and keeps the weights of
// up to four ranks resident (more ranks stream through four slots); four TMEM accumulators form a
// ring; each epilogue warp stages its 32 x 16 block of u and w in shared memory and writes it with
// one TMA store a rank, so no thread issues a global store.
// d = 128 (write_producer_kernel): one CTA per tile, the weights double-buffered per l, u and w
// written by the epilogue threads.
// Every wait is a bounded mbarrier poll that records PRISM_ERR_TIMEOUT in the library's producer
// status word.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "chunk_common.cuh"
#include "producer.cuh"

namespace prism {
namespace {

__device__ uint32_t g_producer_status;

constexpr int PT = 128;                    // tokens per CTA (TMEM lanes, M of the MMA)
constexpr int P_EPI = 8;                   // epilogue warps
constexpr int P_THREADS = 32 * (P_EPI + 1);

// GELU(z) = z Phi(z) with erf from Abramowitz & Stegun, Handbook of Mathematical Functions,
// formula 7.1.26 (absolute error at most 1.5e-7 for x >= 0):
//   erfc(x) ~ t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-x^2),   t = 1 / (1 + p x).
// With x = |z| / sqrt 2 and h = erfc(x) / 2:  Phi(z) = 1 - h for z >= 0 and h for z < 0, so
// GELU(z) = max(z, 0) - |z| h in both cases (no cancellation in the negative tail).  The
// reciprocal and the exponential are the hardware approximations; the rest runs two lanes an
// instruction.  The coefficients below carry the factor 1/2 of h (with a sign flip: the
// polynomial gives -h) and the 1 / sqrt 2 of x.
constexpr float kGeluP = 0.3275911f * 0.70710678118654752f;
constexpr float kGeluA1 = -0.5f * 0.254829592f, kGeluA2 = -0.5f * -0.284496736f,
                kGeluA3 = -0.5f * 1.421413741f, kGeluA4 = -0.5f * -1.453152027f,
                kGeluA5 = -0.5f * 1.061405429f;
constexpr float kGeluE = -0.5f * 1.4426950408889634f;  // exp(-z^2 / 2) = 2^(kGeluE z^2)

__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ unsigned long long pk2(float a, float b) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void upk2(unsigned long long r, float &a, float &b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b, unsigned long long c) {
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b) {
    unsigned long long d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// One residual step on N columns (N even): z = p r, delta = GELU(z), r -= delta, u = bl delta
// (u may alias p).
template <int N>
__device__ __forceinline__ void gelu_step(const float *p, float *r, float bl, float *u) {
    const unsigned long long cA5 = pk2(kGeluA5, kGeluA5), cA4 = pk2(kGeluA4, kGeluA4),
                             cA3 = pk2(kGeluA3, kGeluA3), cA2 = pk2(kGeluA2, kGeluA2),
                             cA1 = pk2(kGeluA1, kGeluA1), cP = pk2(kGeluP, kGeluP),
                             cE = pk2(kGeluE, kGeluE), one = pk2(1.f, 1.f), b2 = pk2(bl, bl);
#pragma unroll
    for (int i = 0; i < N; i += 2) {
        const unsigned long long z = mul2(pk2(p[i], p[i + 1]), pk2(r[i], r[i + 1]));
        float z0, z1;
        upk2(z, z0, z1);
        const unsigned long long az = pk2(fabsf(z0), fabsf(z1));
        float d0, d1;
        upk2(fma2(az, cP, one), d0, d1);
        const unsigned long long t = pk2(rcp_approx(d0), rcp_approx(d1));
        float q0, q1;
        upk2(mul2(mul2(z, cE), z), q0, q1);
        const unsigned long long e = pk2(ex2_approx(q0), ex2_approx(q1));
        unsigned long long s = fma2(t, cA5, cA4);
        s = fma2(t, s, cA3);
        s = fma2(t, s, cA2);
        s = fma2(t, s, cA1);
        const unsigned long long nh = mul2(mul2(s, t), e);                         // -h
        const unsigned long long dl = fma2(az, nh, pk2(fmaxf(z0, 0.f), fmaxf(z1, 0.f)));  // GELU(z)
        float r0, r1, u0, u1;
        upk2(fma2(dl, pk2(-1.f, -1.f), pk2(r[i], r[i + 1])), r0, r1);
        upk2(mul2(b2, dl), u0, u1);
        r[i] = r0;
        r[i + 1] = r1;
        u[i] = u0;
        u[i + 1] = u1;
    }
}

template <int D>
struct ProdLayout {
    static constexpr uint32_t A_BLK = PT * 128;            // 128 token rows x 64 bf16 columns
    static constexpr uint32_t A = 0;                       // anchor hi tile, K-major SW128
    static constexpr uint32_t A_LO = A + A_BLK * (D / 64); // anchor lo tile
    static constexpr uint32_t W_BLK = 2 * D * 128;         // [W_k; W_p] rows of one 64-col block
    static constexpr uint32_t WBUF = W_BLK * (D / 64);
    static constexpr uint32_t W = A_LO + A_BLK * (D / 64); // two weight buffers
    static constexpr uint32_t BYTES = W + 2 * WBUF + 1024;
    static constexpr uint32_t TCOLS = 4 * D <= 256 ? 256 : 512;   // two [k | p] accumulators
    static_assert(BYTES <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ void unpack8(const uint4 &v, float *f) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}

__device__ __forceinline__ uint4 pack8(const float *f) {
    return make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                      pack_bf16(f[6], f[7]));
}

template <int D>
__global__ void __launch_bounds__(P_THREADS, D == 64 ? 2 : 1) write_producer_kernel(ProducerArgs p,
                                                                     const __grid_constant__ CUtensorMap mk,
                                                                     const __grid_constant__ CUtensorMap mp) {
    using LY = ProdLayout<D>;
    constexpr int HALF = D / 2;  // columns of an epilogue thread
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t wbar[2], full[2], tfree[2], a_ready, drain;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int failed_sh;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = blockIdx.x * PT, h = blockIdx.y, b = blockIdx.z;
    const int T = p.T, H = p.H, L = p.L;
    const uint32_t sb = smem_u32(sm);
    uint32_t *status = &g_producer_status;
    const uint32_t lim = p.stall ? kStallTestPolls : kWaitPolls;

    if (warp == P_EPI) tmem_alloc(&tmem_base_sh, LY::TCOLS);
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&wbar[i], 1);
            mbar_init(&full[i], 1);
            mbar_init(&tfree[i], P_EPI);
        }
        mbar_init(&a_ready, P_EPI);
        mbar_init(&drain, 1);
        mbar_fence_init();
        failed_sh = 0;
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tb = tmem_base_sh;

    if (warp == P_EPI) {
        // ---------------- weights by TMA, one MMA per rank ----------------
        if (lane == 0) {
            auto load_w = [&](int l) {  // [W_k^(l); W_p^(l)] into buffer l % 2
                const int bi = l & 1;
                uint8_t *dst = sm + LY::W + bi * LY::WBUF;
                mbar_expect_tx(&wbar[bi], LY::WBUF);
                for (int blk = 0; blk < D / 64; ++blk) {
                    tma_load_4d(dst + blk * LY::W_BLK, &mk, blk * 64, 0, l, h, &wbar[bi]);
                    tma_load_4d(dst + blk * LY::W_BLK + D * 128, &mp, blk * 64, 0, l, h, &wbar[bi]);
                }
            };
            int issued = 0;
            if (!p.stall)
                for (; issued < L && issued < 2; ++issued) load_w(issued);
            bool ok = mbar_wait(&a_ready, 0, status, lim);
            const uint32_t id = idesc_bf16(128, 2 * D, 0, 0);
            auto oa = [](int ks) { return (uint64_t)koff_k_sw128(ks, LY::A_BLK); };
            auto ow = [](int ks) { return (uint64_t)koff_k_sw128(ks, LY::W_BLK); };
            const uint64_t dA = make_desc(sb + LY::A, 16, 1024, 2);
            const uint64_t dAl = make_desc(sb + LY::A_LO, 16, 1024, 2);
            for (int l = 0; l < L && ok; ++l) {
                const int bi = l & 1;
                if (!mbar_wait(&wbar[bi], (l >> 1) & 1, status, lim)) { ok = false; break; }
                // the epilogue of rank l - 2 has read this accumulator
                if (l >= 2 && !mbar_wait(&tfree[bi], ((l - 2) >> 1) & 1, status, lim)) { ok = false; break; }
                fence_after_sync();
                const uint64_t dW = make_desc(sb + LY::W + bi * LY::WBUF, 16, 1024, 2);
                // the anchor as a bf16 hi / lo pair: (a_hi + a_lo) W^T, the weights exact bf16
                mma_steps<D / 16>(tb + bi * 2 * D, id, dA, dW, oa, ow, false);
                mma_steps<D / 16>(tb + bi * 2 * D, id, dAl, dW, oa, ow, true);
                mma_commit(&full[bi]);
                if (issued < L) {  // W of rank l + 2 into this buffer once the MMA has read it
                    if (!mbar_wait(&full[bi], (l >> 1) & 1, status, lim)) { ok = false; break; }
                    load_w(issued++);
                }
            }
            if (!ok) failed_sh = 1;
            mma_commit(&drain);
            mbar_wait(&drain, 0, nullptr, lim);
            // after a failure, weight loads still in flight land before the CTA exits
            if (!ok)
                for (int l = issued > 2 ? issued - 2 : 0; l < issued; ++l)
                    mbar_wait(&wbar[l & 1], (l >> 1) & 1, nullptr, kStallTestPolls);
        }
    } else {
        // ---------------- anchor, then the residual chain, rank by rank ----------------
        const int q = warp & 3, hs = warp >> 2;  // TMEM lane quarter, column half
        const int row = 32 * q + lane, t = t0 + row;
        const bool live = t < T;
        const int c_base = hs * HALF;
        const size_t tok = ((size_t)b * T + t) * H + h;
        const __nv_bfloat16 *x = (const __nv_bfloat16 *)p.x;
        const __nv_bfloat16 *v = (const __nv_bfloat16 *)p.v;
        float r[HALF];
#pragma unroll
        for (int c8 = 0; c8 < HALF; c8 += 8) {
            const int col = c_base + c8;
            float a8[8], xf[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) a8[i] = 0.f;
            if (live) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (t - j >= 0) {
                        const uint4 xv = *reinterpret_cast<const uint4 *>(x + (((size_t)b * T + t - j) * H + h) * D + col);
                        unpack8(xv, xf);
                        const float *cj = p.conv + ((size_t)h * 4 + j) * D + col;
                        const float4 c0 = *reinterpret_cast<const float4 *>(cj);
                        const float4 c1 = *reinterpret_cast<const float4 *>(cj + 4);
                        const float cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                        for (int i = 0; i < 8; ++i) a8[i] = fmaf(cw[i], xf[i], a8[i]);
                    }
                }
                unpack8(*reinterpret_cast<const uint4 *>(v + tok * D + col), r + c8);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) r[c8 + i] = 0.f;
            }
            uint4 hi, lo;
            split8(a8, hi, lo);
            const uint32_t off = sw128_off(row, col, LY::A_BLK);
            st16(sm + LY::A, off, hi);
            st16(sm + LY::A_LO, off, lo);
        }
        fence_async_smem();
        fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_ready);

        __nv_bfloat16 *uo = (__nv_bfloat16 *)p.u, *wo = (__nv_bfloat16 *)p.w;
        bool ok = true;
        for (int l = 0; l < L && ok; ++l) {
            const int bi = l & 1;
            if (!mbar_wait(&full[bi], (l >> 1) & 1, status, lim)) { ok = false; break; }
            fence_after_sync();
            const float bl = live ? p.beta[tok * L + l] : 0.f;
            const size_t orow = (tok * L + l) * D;
            // 16 columns at a time (directions, then gains), few registers beyond the residual
#pragma unroll
            for (int ci = 0; ci < HALF / 16; ++ci) {
                const int col = c_base + 16 * ci;
                float kk[16];
                tmem_ld16(taddr(tb, 32 * q, bi * 2 * D + col), kk);
                tmem_wait_ld();
                if (live) {
                    *reinterpret_cast<uint4 *>(wo + orow + col) = pack8(kk);
                    *reinterpret_cast<uint4 *>(wo + orow + col + 8) = pack8(kk + 8);
                }
                float pp[16];
                tmem_ld16(taddr(tb, 32 * q, bi * 2 * D + D + col), pp);
                tmem_wait_ld();
                gelu_step<16>(pp, r + 16 * ci, bl, pp);
                if (live) {
                    *reinterpret_cast<uint4 *>(uo + orow + col) = pack8(pp);
                    *reinterpret_cast<uint4 *>(uo + orow + col + 8) = pack8(pp + 8);
                }
            }
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tfree[bi]);
        }
        if (!ok) failed_sh = 1;
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == P_EPI) tmem_dealloc(tb, LY::TCOLS);
}

// ------------------------------------------------------------------------------------------------
// d = 64: the persistent producer

constexpr int RCW = 16;    // columns of one epilogue thread
constexpr int RNW = 4;     // weight slots, one rank's [W_k; W_p] each
constexpr int RNACC = 4;   // TMEM accumulators, one rank's [k | p] each

template <int D>
struct RingLayout {
    static constexpr int NCS = D / RCW;                     // column slices
    static constexpr int EPI = 4 * NCS;                     // epilogue warps (TMEM lane quarter x slice)
    static constexpr int LOADW = EPI, MMAW = EPI + 1;       // the load warp, the MMA warp
    static constexpr int THREADS = 32 * (EPI + 2);
    static constexpr uint32_t A_BLK = PT * 128;
    static constexpr uint32_t A = 0, A_LO = A_BLK;          // anchor hi / lo, K-major SW128
    static constexpr int XROWS = PT + 3;                    // x rows t0 - 3 .. t0 + PT - 1
    static constexpr uint32_t X = 2 * A_BLK;                // SW128 rows of 128 bytes
    static constexpr uint32_t X_BYTES = XROWS * 128;
    static constexpr uint32_t V = (X + X_BYTES + 1023) / 1024 * 1024;
    static constexpr uint32_t V_BYTES = PT * 128;
    static constexpr uint32_t WSLOT = 2 * D * 128;          // [W_k; W_p] of one rank, K-major SW128
    static constexpr uint32_t W = V + V_BYTES;
    static constexpr uint32_t BOX = 32 * RCW * 2;           // one warp's 32 rows x 16 columns (SW32)
    static constexpr uint32_t OUT = W + RNW * WSLOT;        // [warp][buffer][w, u]
    static constexpr uint32_t BYTES = OUT + EPI * 4 * BOX + 1024;
    static_assert(D == 64, "one 64-column block per row");
    static_assert(BYTES <= 227 * 1024, "shared memory budget");
    static_assert(RNACC * 2 * D <= 512, "TMEM columns");
};

struct RingMaps {
    CUtensorMap x, v, wk, wp, u, w;
};

template <int D>
__global__ void __launch_bounds__(RingLayout<D>::THREADS, 1)
    write_producer_ring_kernel(ProducerArgs p, const __grid_constant__ RingMaps maps, long long ntiles) {
    using LY = RingLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t xv_full, xv_free, a_ready, drain;
    __shared__ uint64_t w_full[RNW], w_free[RNW], acc_full[RNACC], acc_free[RNACC];
    __shared__ uint32_t tmem_base_sh;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = p.T, H = p.H, B = p.B, L = p.L;
    const long long nt = (T + PT - 1) / PT;  // tiles per sequence
    // this CTA's contiguous range of tiles; tile n = (h * B + b) * nt + j
    const long long n0 = ntiles * blockIdx.x / gridDim.x, n1 = ntiles * (blockIdx.x + 1) / gridDim.x;
    const bool resident = L <= RNW;  // the weights of all ranks stay in their slots per head
    const uint32_t sb = smem_u32(sm);
    uint32_t *status = &g_producer_status;
    const uint32_t lim = p.stall ? kStallTestPolls : kWaitPolls;

    if (warp == LY::MMAW) tmem_alloc(&tmem_base_sh, 512);
    if (tid == 0) {
        mbar_init(&xv_full, 1);
        mbar_init(&xv_free, LY::EPI);
        mbar_init(&a_ready, LY::EPI);
        mbar_init(&drain, 1);
        for (int i = 0; i < RNW; ++i) {
            mbar_init(&w_full[i], 1);
            mbar_init(&w_free[i], 1);
        }
        for (int i = 0; i < RNACC; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_free[i], LY::EPI);
        }
        mbar_fence_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tb = tmem_base_sh;

    if (warp == LY::LOADW) {
        // ---------------- x and v rows of each tile; the weights ----------------
        if (lane == 0 && !p.stall) {
            int epoch = -1, prev_h = -1;
            long long k = 0;
            uint32_t wfills[RNW] = {0, 0, 0, 0};  // loads issued into each weight slot
            bool ok = true;
            auto load_w = [&](int slot, int h, int l) {
                uint8_t *dst = sm + LY::W + slot * LY::WSLOT;
                mbar_expect_tx(&w_full[slot], LY::WSLOT);
                tma_load_4d(dst, &maps.wk, 0, 0, l, h, &w_full[slot]);
                tma_load_4d(dst + D * 128, &maps.wp, 0, 0, l, h, &w_full[slot]);
                ++wfills[slot];
            };
            for (long long n = n0; n < n1 && ok; ++n, ++k) {
                const int j = (int)(n % nt), bh = (int)(n / nt), b = bh % B, h = bh / B;
                if (k >= 1 && !mbar_wait(&xv_free, (uint32_t)((k - 1) & 1), status, lim)) { ok = false; break; }
                mbar_expect_tx(&xv_full, LY::X_BYTES + LY::V_BYTES);
                tma_load_4d(sm + LY::X, &maps.x, 0, h, j * PT - 3, b, &xv_full);
                tma_load_4d(sm + LY::V, &maps.v, 0, h, j * PT, b, &xv_full);
                if (resident) {
                    if (h == prev_h) continue;
                    prev_h = h;
                    ++epoch;
                    for (int l = 0; l < L && ok; ++l) {
                        if (epoch >= 1 && !mbar_wait(&w_free[l], (uint32_t)((epoch - 1) & 1), status, lim)) ok = false;
                        else load_w(l, h, l);
                    }
                } else {
                    for (int l = 0; l < L && ok; ++l) {
                        const long long use = k * L + l;
                        const int slot = (int)(use % RNW);
                        const long long f = use / RNW;
                        if (f >= 1 && !mbar_wait(&w_free[slot], (uint32_t)((f - 1) & 1), status, lim)) ok = false;
                        else load_w(slot, h, l);
                    }
                }
            }
            // loads still in flight land before the CTA exits (in a normal run every one has
            // been waited for by its consumer already)
            if (k > 0) mbar_wait(&xv_full, (uint32_t)((k - 1) & 1), nullptr, lim);
            for (int i = 0; i < RNW; ++i)
                if (wfills[i]) mbar_wait(&w_full[i], (wfills[i] - 1) & 1, nullptr, lim);
        }
    } else if (warp == LY::MMAW) {
        // ---------------- one M = 128, N = 2d MMA pair (anchor hi, lo) per rank ----------------
        if (lane == 0) {
            const uint32_t id = idesc_bf16(128, 2 * D, 0, 0);
            auto oa = [](int ks) { return (uint64_t)koff_k_sw128(ks, LY::A_BLK); };
            auto ow = [](int ks) { return (uint64_t)koff_k_sw128(ks, LY::WSLOT); };
            const uint64_t dA = make_desc(sb + LY::A, 16, 1024, 2);
            const uint64_t dAl = make_desc(sb + LY::A_LO, 16, 1024, 2);
            int epoch = -1, prev_h = -1;
            long long k = 0, g = 0;
            bool ok = true;
            for (long long n = n0; n < n1 && ok; ++n, ++k) {
                const int h = (int)(n / nt) / B;
                if (h != prev_h) {
                    prev_h = h;
                    ++epoch;
                }
                // the last of this CTA's tiles on this head releases the resident weights
                const bool last_of_head = n + 1 == n1 || (int)((n + 1) / nt) / B != h;
                if (!mbar_wait(&a_ready, (uint32_t)(k & 1), status, lim)) { ok = false; break; }
                for (int l = 0; l < L; ++l, ++g) {
                    const long long use = k * L + l;
                    const int ws = resident ? l : (int)(use % RNW);
                    const uint32_t wpar = resident ? (uint32_t)(epoch & 1) : (uint32_t)((use / RNW) & 1);
                    const int slot = (int)(g % RNACC);
                    if (!mbar_wait(&w_full[ws], wpar, status, lim) ||
                        (g >= RNACC && !mbar_wait(&acc_free[slot], (uint32_t)((g / RNACC - 1) & 1), status, lim))) {
                        ok = false;
                        break;
                    }
                    fence_after_sync();
                    const uint64_t dW = make_desc(sb + LY::W + ws * LY::WSLOT, 16, 1024, 2);
                    const uint32_t acc = tb + slot * 2 * D;
                    mma_steps<D / 16>(acc, id, dA, dW, oa, ow, false);
                    mma_steps<D / 16>(acc, id, dAl, dW, oa, ow, true);
                    mma_commit(&acc_full[slot]);
                    if (!resident || last_of_head) mma_commit(&w_free[ws]);
                }
            }
            mma_commit(&drain);
            mbar_wait(&drain, 0, nullptr, lim);
        }
    } else {
        // ---------------- anchor, residual chain, staged TMA stores ----------------
        const int q = warp & 3, cs = warp >> 2;  // TMEM lane quarter, column slice
        const int row = 32 * q + lane, col0 = cs * RCW;
        uint8_t *ob = sm + LY::OUT + warp * 4 * LY::BOX;  // [buffer][w, u]
        long long k = 0, g = 0;
        bool ok = true;
        for (long long n = n0; n < n1 && ok; ++n, ++k) {
            const int j = (int)(n % nt), bh = (int)(n / nt), b = bh % B, h = bh / B;
            const int t0 = j * PT, t = t0 + row;
            const bool live = t < T;
            const size_t tok = ((size_t)b * T + t) * H + h;
            // ShortConv taps of this head (broadcast loads, L1 hits after the first tile)
            float a[RCW], r[RCW];
#pragma unroll
            for (int i = 0; i < RCW; ++i) a[i] = 0.f;
            if (!mbar_wait(&xv_full, (uint32_t)(k & 1), status, lim)) { ok = false; break; }
#pragma unroll
            for (int tap = 0; tap < 4; ++tap) {
                const float *cj = p.conv + ((size_t)h * 4 + tap) * D + col0;
                const int xr = row + 3 - tap;  // x stage row of token t - tap
#pragma unroll
                for (int c8 = 0; c8 < RCW / 8; ++c8) {
                    const int chunk = (col0 >> 3) + c8;
                    float xf[8];
                    unpack8(*reinterpret_cast<const uint4 *>(sm + LY::X + xr * 128 + ((chunk ^ (xr & 7)) << 4)), xf);
                    const float4 c0 = *reinterpret_cast<const float4 *>(cj + 8 * c8);
                    const float4 c1 = *reinterpret_cast<const float4 *>(cj + 8 * c8 + 4);
                    const float cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                    for (int i = 0; i < 8; ++i) a[8 * c8 + i] = fmaf(cw[i], xf[i], a[8 * c8 + i]);
                }
            }
#pragma unroll
            for (int c8 = 0; c8 < RCW / 8; ++c8) {
                const int chunk = (col0 >> 3) + c8;
                unpack8(*reinterpret_cast<const uint4 *>(sm + LY::V + row * 128 + ((chunk ^ (row & 7)) << 4)), r + 8 * c8);
                uint4 hi, lo;
                split8(a + 8 * c8, hi, lo);
                const uint32_t off = sw128_off(row, col0 + 8 * c8, LY::A_BLK);
                st16(sm + LY::A, off, hi);
                st16(sm + LY::A_LO, off, lo);
            }
            fence_async_smem();
            fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&a_ready);
                mbar_arrive(&xv_free);
            }
            float bl = live ? p.beta[tok * L] : 0.f;
            for (int l = 0; l < L; ++l, ++g) {
                const int slot = (int)(g % RNACC);
                if (!mbar_wait(&acc_full[slot], (uint32_t)((g / RNACC) & 1), status, lim)) { ok = false; break; }
                fence_after_sync();
                float kk[RCW], pp[RCW];
                tmem_ld16(taddr(tb, 32 * q, slot * 2 * D + col0), kk);
                tmem_ld16(taddr(tb, 32 * q, slot * 2 * D + D + col0), pp);
                tmem_wait_ld();
                fence_before_sync();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&acc_free[slot]);
                    if (g >= 2) bulk_wait_read_n<1>();  // the stores of rank g - 2 have read this buffer
                }
                const float bcur = bl;
                if (l + 1 < L && live) bl = p.beta[tok * L + l + 1];
                __syncwarp();
                uint8_t *bw = ob + (uint32_t)(g & 1) * 2 * LY::BOX, *bu = bw + LY::BOX;
                const int sw = (lane >> 2) & 1;  // SW32: the 16-byte chunk index XOR row bit 2
                st16(bw, lane * 32 + ((0 ^ sw) << 4), pack8(kk));
                st16(bw, lane * 32 + ((1 ^ sw) << 4), pack8(kk + 8));
                gelu_step<RCW>(pp, r, bcur, pp);
                st16(bu, lane * 32 + ((0 ^ sw) << 4), pack8(pp));
                st16(bu, lane * 32 + ((1 ^ sw) << 4), pack8(pp + 8));
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_5d(&maps.w, bw, col0, l, h, t0 + 32 * q, b);
                    tma_store_5d(&maps.u, bu, col0, l, h, t0 + 32 * q, b);
                    bulk_commit();
                }
            }
        }
        if (lane == 0) bulk_wait_all();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == LY::MMAW) tmem_dealloc(tb, 512);
}

// The driver's tensor-map encoder, fetched once through the runtime (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 4-D map over bf16 weights [H, L, d, d] (row = output index): dims {d_in, d_out, L, H}, box
// {64, d, 1, 1} (one 64-column block of one (h, l) matrix).
bool weight_map(CUtensorMap *m, const void *base, int H, int L, int d) {
    auto enc = map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)d, (cuuint64_t)L, (cuuint64_t)H};
    const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)d * d * 2, (cuuint64_t)L * d * d * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)d, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// x or v [B,T,H,d] bf16 as a 4-D map {d, H, T, B}; box {64, 1, rows, 1}, 128-byte swizzle.
bool act_map(CUtensorMap *m, const void *base, int B, int T, int H, int d, int rows) {
    auto enc = map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)T * H * d * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// u or w [B,T,H,L,d] bf16 as a 5-D map {d, L, H, T, B}; box {16, 1, 1, 32, 1} (one epilogue
// warp's block of one rank), 32-byte swizzle.
bool out_map(CUtensorMap *m, void *base, int B, int T, int H, int L, int d) {
    auto enc = map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)L, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[4] = {(cuuint64_t)d * 2, (cuuint64_t)L * d * 2, (cuuint64_t)H * L * d * 2,
                                   (cuuint64_t)T * H * L * d * 2};
    const cuuint32_t box[5] = {RCW, 1, 1, 32, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, base, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int device_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
        return 1;
    return n;
}

cudaError_t launch_producer_ring(const ProducerArgs &a, cudaStream_t s) {
    constexpr int D = 64;
    using LY = RingLayout<D>;
    RingMaps maps;
    if (!act_map(&maps.x, a.x, a.B, a.T, a.H, D, LY::XROWS) || !act_map(&maps.v, a.v, a.B, a.T, a.H, D, PT) ||
        !weight_map(&maps.wk, a.Wk, a.H, a.L, D) || !weight_map(&maps.wp, a.Wp, a.H, a.L, D) ||
        !out_map(&maps.u, a.u, a.B, a.T, a.H, a.L, D) || !out_map(&maps.w, a.w, a.B, a.T, a.H, a.L, D))
        return cudaErrorInvalidValue;
    auto kern = write_producer_ring_kernel<D>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)LY::BYTES);
    if (err != cudaSuccess) return err;
    const long long ntiles = (long long)a.H * a.B * ((a.T + PT - 1) / PT);
    const int grid = (int)std::min<long long>(ntiles, device_sms());
    launch_probe_mark(s);
    kern<<<grid, LY::THREADS, LY::BYTES, s>>>(a, maps, ntiles);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_producer_t(const ProducerArgs &a, cudaStream_t s) {
    CUtensorMap mk, mp;
    if (!weight_map(&mk, a.Wk, a.H, a.L, D) || !weight_map(&mp, a.Wp, a.H, a.L, D))
        return cudaErrorInvalidValue;
    using LY = ProdLayout<D>;
    auto kern = write_producer_kernel<D>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)LY::BYTES);
    if (err != cudaSuccess) return err;
    dim3 grid((a.T + PT - 1) / PT, a.H, a.B);
    launch_probe_mark(s);
    kern<<<grid, P_THREADS, LY::BYTES, s>>>(a, mk, mp);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_write_producer(const ProducerArgs &a, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    return a.d == 128 ? launch_producer_t<128>(a, s) : launch_producer_ring(a, s);
}

// Read and clear the producer's status word (PRISM_OK or PRISM_ERR_TIMEOUT).
cudaError_t producer_status(uint32_t *out) {
    uint32_t word = 0;
    cudaError_t err = cudaMemcpyFromSymbol(&word, g_producer_status, sizeof word);
    if (err != cudaSuccess) return err;
    if (word != 0) {
        const uint32_t zero = 0;
        if ((err = cudaMemcpyToSymbol(g_producer_status, &zero, sizeof zero)) != cudaSuccess) return err;
    }
    *out = word;
    return cudaSuccess;
}

}  // namespace prism
