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
// One kernel (write_producer_ring_kernel), persistent: one CTA per SM walks a contiguous range of
// 128-token tiles of one (batch, head) at a time (head-major order, so a CTA's tiles share their
// weights).  Its epilogue warps build the anchor tile (the A operand, as a bf16 hi / lo pair: a
// single bf16 anchor lets the residual chain amplify its rounding past the bf16 output tolerance by
// the fourth rank) and hold the residual in registers (one token row, 16 columns a thread); one
// thread issues, for each l, one M = 128, N = 128 MMA pair of the anchor against the stacked
// weights into one of four TMEM accumulators, so the MMA of rank l + 1 runs while the epilogue of
// rank l reads k^(l) and p^(l), applies the GELU step and writes u and w.  A load warp brings each
// tile's x rows (with the 3-token causal halo; rows before the sequence start read as zeros) by TMA
// into swizzled shared memory while the previous tile is in its epilogue, and keeps the weights of
// up to NW ranks resident (more ranks stream through NW slots).  Each epilogue warp stages its
// 32 x 16 blocks of w and u in shared memory and writes each with one TMA store, so no thread
// issues a global store.  At d = 128 the two CTAs of a pair take one 64-column half of k, p, u, w
// each (the residual chain is column-wise); both build the whole anchor (the MMA's K).
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

constexpr int PT = 128;                    // tokens per tile (TMEM lanes, M of the MMA)

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

// 5-D tiled TMA store of one box from shared memory (rows outside the tensor are not written),
// in this thread's current bulk group.
__device__ __forceinline__ void tma_store_5d(const void *tmap, const void *src, int x, int y, int z, int w,
                                             int v) {
    asm volatile(
        "cp.async.bulk.tensor.5d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3, %4, %5}], [%6];"
        ::"l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(v), "r"(smem_u32(src))
        : "memory");
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

// ------------------------------------------------------------------------------------------------
// The persistent producer.  Each CTA writes 64 output columns of every token of its tiles: all of
// them at d = 64; at d = 128 the two CTAs of a pair split the columns (the residual chain is
// column-wise, so the halves are independent; both build the whole anchor, which is the MMA's K).

constexpr int RCW = 16;    // output columns of one epilogue thread
constexpr int RNACC = 4;   // TMEM accumulators, one rank's [k | p] (128 columns) each

template <int D>
struct RingLayout {
    static constexpr int HALVES = D / 64;                   // CTAs per tile
    static constexpr int NH = 64;                           // output columns of a CTA
    static constexpr int EPI = 4 * (NH / RCW);              // epilogue warps (TMEM lane quarter x slice)
    static constexpr int ACW = D / 4;                       // anchor columns of an epilogue thread
    static constexpr int LOADW = EPI, MMAW = EPI + 1;       // the load warp, the MMA warp
    static constexpr int THREADS = 32 * (EPI + 2);
    static constexpr int NW = D == 64 ? 4 : 2;              // weight slots (one rank's half of [W_k; W_p])
    static constexpr int NBOX = D == 64 ? 4 : 3;            // output staging boxes of a warp (a ring)
    static constexpr uint32_t A_BLK = PT * 128;             // 128 rows x 64 bf16 columns
    static constexpr uint32_t A = 0, A_LO = A_BLK * HALVES; // anchor hi / lo, K-major SW128
    static constexpr int XROWS = PT + 3;                    // x rows t0 - 3 .. t0 + PT - 1
    static constexpr uint32_t XBOX_TX = XROWS * 128;        // one 64-column box of x rows (SW128)
    static constexpr uint32_t XBOX = (XBOX_TX + 1023) / 1024 * 1024;
    static constexpr uint32_t X = 2 * A_BLK * HALVES;
    static constexpr uint32_t V = X + HALVES * XBOX;        // v rows (d = 64 only; SW128)
    static constexpr uint32_t V_BYTES = D == 64 ? PT * 128 : 0;
    static constexpr uint32_t WBLK = 2 * NH * 128;          // [W_k; W_p] rows of one 64-column K block
    static constexpr uint32_t WSLOT = WBLK * HALVES;
    static constexpr uint32_t W = V + V_BYTES;
    static constexpr uint32_t BOX = 32 * RCW * 2;           // one warp's 32 rows x 16 columns (SW32)
    static constexpr uint32_t OUT = W + NW * WSLOT;         // [warp][box]
    static constexpr uint32_t BYTES = OUT + EPI * NBOX * BOX + 1024;
    static constexpr uint32_t XV_TX = HALVES * XBOX_TX + V_BYTES;
    static_assert(D == 64 || D == 128, "widths");
    static_assert(BYTES <= 227 * 1024, "shared memory budget");
    static_assert(RNACC * 2 * NH <= 512, "TMEM columns");
};

struct RingMaps {
    CUtensorMap x, v, wk, wp, u, w;
};

// Walks tiles n0, n0 + 1, ... of the head-major order n = (h B + b) nt + j with 32-bit steps.
struct TileWalk {
    int j, bh, left;  // tile within its sequence, sequence index h B + b, tiles still to visit
    int nt, B;
    __device__ TileWalk(long long n0, long long n1, int nt_, int B_) : nt(nt_), B(B_) {
        j = (int)(n0 % nt_);
        bh = (int)(n0 / nt_);
        left = (int)(n1 - n0);
    }
    __device__ bool more() const { return left > 0; }
    __device__ void next() {
        --left;
        if (++j == nt) {
            j = 0;
            ++bh;
        }
    }
    __device__ int b() const { return bh % B; }
    __device__ int h() const { return bh / B; }
    // the next tile (if any) belongs to another head
    __device__ bool last_of_head() const { return left == 1 || (j + 1 == nt && (bh + 1) / B != bh / B); }
};

template <int D>
__global__ void __launch_bounds__(RingLayout<D>::THREADS, 1)
    write_producer_ring_kernel(ProducerArgs p, const __grid_constant__ RingMaps maps, long long ntiles) {
    using LY = RingLayout<D>;
    constexpr int NW = LY::NW, NH = LY::NH;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t xv_full, xv_free, a_ready, drain;
    __shared__ uint64_t w_full[NW], w_free[NW], acc_full[RNACC], acc_free[RNACC];
    __shared__ uint32_t tmem_base_sh;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = p.T, H = p.H, B = p.B, L = p.L;
    const int half = blockIdx.x % LY::HALVES;  // which 64 output columns
    const long long G = gridDim.x / LY::HALVES, pid = blockIdx.x / LY::HALVES;
    const int nt = (T + PT - 1) / PT;  // tiles per sequence
    // this CTA's contiguous range of tiles; tile n = (h * B + b) * nt + j
    const long long n0 = ntiles * pid / G, n1 = ntiles * (pid + 1) / G;
    const bool resident = L <= NW;  // the weights of all ranks stay in their slots per head
    const uint32_t sb = smem_u32(sm);
    uint32_t *status = &g_producer_status;
    const uint32_t lim = p.stall ? kStallTestPolls : kWaitPolls;

    if (warp == LY::MMAW) tmem_alloc(&tmem_base_sh, 512);
    if (tid == 0) {
        mbar_init(&xv_full, 1);
        mbar_init(&xv_free, LY::EPI);
        mbar_init(&a_ready, LY::EPI);
        mbar_init(&drain, 1);
        for (int i = 0; i < NW; ++i) {
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
        // ---------------- x (and v) rows of each tile; the weights ----------------
        if (lane == 0 && !p.stall) {
            int epoch = -1, prev_h = -1, k = 0;
            uint32_t wfills[NW] = {};  // loads issued into each weight slot
            bool ok = true;
            auto load_w = [&](int slot, int h, int l) {
                uint8_t *dst = sm + LY::W + slot * LY::WSLOT;
                mbar_expect_tx(&w_full[slot], LY::WSLOT);
#pragma unroll
                for (int kb = 0; kb < LY::HALVES; ++kb) {
                    tma_load_4d(dst + kb * LY::WBLK, &maps.wk, kb * 64, half * NH, l, h, &w_full[slot]);
                    tma_load_4d(dst + kb * LY::WBLK + NH * 128, &maps.wp, kb * 64, half * NH, l, h, &w_full[slot]);
                }
#pragma unroll
                for (int i = 0; i < NW; ++i) wfills[i] += i == slot;
            };
            for (TileWalk tw(n0, n1, nt, B); tw.more() && ok; tw.next(), ++k) {
                const int j = tw.j, b = tw.b(), h = tw.h();
                if (k >= 1 && !mbar_wait(&xv_free, (uint32_t)((k - 1) & 1), status, lim)) { ok = false; break; }
                mbar_expect_tx(&xv_full, LY::XV_TX);
#pragma unroll
                for (int xb = 0; xb < LY::HALVES; ++xb)
                    tma_load_4d(sm + LY::X + xb * LY::XBOX, &maps.x, xb * 64, h, j * PT - 3, b, &xv_full);
                if constexpr (D == 64) tma_load_4d(sm + LY::V, &maps.v, 0, h, j * PT, b, &xv_full);
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
                        const uint32_t use = (uint32_t)k * L + l;
                        const int slot = (int)(use % NW);
                        const uint32_t f = use / NW;
                        if (f >= 1 && !mbar_wait(&w_free[slot], (uint32_t)((f - 1) & 1), status, lim)) ok = false;
                        else load_w(slot, h, l);
                    }
                }
            }
            // loads still in flight land before the CTA exits (in a normal run every one has
            // been waited for by its consumer already)
            if (k > 0) mbar_wait(&xv_full, (uint32_t)((k - 1) & 1), nullptr, lim);
#pragma unroll
            for (int i = 0; i < NW; ++i)
                if (wfills[i]) mbar_wait(&w_full[i], (wfills[i] - 1) & 1, nullptr, lim);
        }
    } else if (warp == LY::MMAW) {
        // ---------------- one M = 128, N = 128 MMA pair (anchor hi, lo) per rank ----------------
        if (lane == 0) {
            const uint32_t id = idesc_bf16(128, 2 * NH, 0, 0);
            auto oa = [](int ks) { return (uint64_t)koff_k_sw128(ks, LY::A_BLK); };
            auto ow = [](int ks) { return (uint64_t)koff_k_sw128(ks, LY::WBLK); };
            const uint64_t dA = make_desc(sb + LY::A, 16, 1024, 2);
            const uint64_t dAl = make_desc(sb + LY::A_LO, 16, 1024, 2);
            int epoch = -1, prev_h = -1;
            uint32_t k = 0, g = 0;
            bool ok = true;
            for (TileWalk tw(n0, n1, nt, B); tw.more() && ok; tw.next(), ++k) {
                const int h = tw.h();
                if (h != prev_h) {
                    prev_h = h;
                    ++epoch;
                }
                // the last of this CTA's tiles on this head releases the resident weights
                const bool last_of_head = tw.last_of_head();
                if (!mbar_wait(&a_ready, (uint32_t)(k & 1), status, lim)) { ok = false; break; }
                for (int l = 0; l < L; ++l, ++g) {
                    const uint32_t use = k * L + l;
                    const int ws = resident ? l : (int)(use % NW);
                    const uint32_t wpar = resident ? (uint32_t)(epoch & 1) : (uint32_t)((use / NW) & 1);
                    const int slot = (int)(g % RNACC);
                    if (!mbar_wait(&w_full[ws], wpar, status, lim) ||
                        (g >= RNACC && !mbar_wait(&acc_free[slot], (uint32_t)((g / RNACC - 1) & 1), status, lim))) {
                        ok = false;
                        break;
                    }
                    fence_after_sync();
                    const uint64_t dW = make_desc(sb + LY::W + ws * LY::WSLOT, 16, 1024, 2);
                    const uint32_t acc = tb + slot * 2 * NH;
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
        const int row = 32 * q + lane, col0 = cs * RCW, ocol = half * NH + col0;
        uint8_t *ob = sm + LY::OUT + warp * LY::NBOX * LY::BOX;
        const __nv_bfloat16 *vg = (const __nv_bfloat16 *)p.v;
        const int sw = (lane >> 2) & 1;  // SW32 staging: the 16-byte chunk index XOR row bit 2
        uint4 vnext[2] = {};             // d = 128: the next tile's v columns, loaded a rank ahead
        auto load_v = [&](int j, int b, int h) {
            const int t = j * PT + row;
            if (t < T) {
                const uint4 *src = reinterpret_cast<const uint4 *>(vg + (((size_t)b * T + t) * H + h) * D + ocol);
                vnext[0] = src[0];
                vnext[1] = src[1];
            } else {
                vnext[0] = vnext[1] = make_uint4(0, 0, 0, 0);
            }
        };
        if constexpr (D != 64)
            if (n0 < n1) {
                const TileWalk tw(n0, n1, nt, B);
                load_v(tw.j, tw.b(), tw.h());
            }
        uint32_t k = 0, g = 0, m = 0;  // tiles, ranks, staging boxes of this thread so far
        bool ok = true;
        auto box = [&]() {  // the next staging box, once its previous store has read it
            if (lane == 0 && m >= LY::NBOX) bulk_wait_read_n<LY::NBOX - 1>();
            __syncwarp();
            return ob + (uint32_t)(m % LY::NBOX) * LY::BOX;
        };
        auto put = [&](uint8_t *bx, const float *v16, const CUtensorMap *map, int l, int h, int t0, int b) {
            st16(bx, lane * 32 + ((0 ^ sw) << 4), pack8(v16));
            st16(bx, lane * 32 + ((1 ^ sw) << 4), pack8(v16 + 8));
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_5d(map, bx, ocol, l, h, t0 + 32 * q, b);
                bulk_commit();
            }
            ++m;
        };
        for (TileWalk tw(n0, n1, nt, B); tw.more() && ok; tw.next(), ++k) {
            const int j = tw.j, b = tw.b(), h = tw.h();
            const int t0 = j * PT, t = t0 + row;
            const bool live = t < T;
            const size_t tok = ((size_t)b * T + t) * H + h;
            float r[RCW];
            if (!mbar_wait(&xv_full, (uint32_t)(k & 1), status, lim)) { ok = false; break; }
            // the anchor's columns [cs ACW, (cs + 1) ACW) of this token row, 16 at a time
#pragma unroll
            for (int a16 = 0; a16 < LY::ACW / 16; ++a16) {
                const int acol = cs * LY::ACW + 16 * a16, xb = acol >> 6;
                float a[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) a[i] = 0.f;
#pragma unroll 1  // (unrolled, the taps' loads are all hoisted and spill)
                for (int tap = 0; tap < 4; ++tap) {
                    // ShortConv taps of this head (broadcast loads, L1 hits after the first tile)
                    const float *cj = p.conv + ((size_t)h * 4 + tap) * D + acol;
                    const int xr = row + 3 - tap;  // x stage row of token t - tap
#pragma unroll
                    for (int c8 = 0; c8 < 2; ++c8) {
                        const int chunk = ((acol & 63) >> 3) + c8;
                        float xf[8];
                        unpack8(*reinterpret_cast<const uint4 *>(sm + LY::X + xb * LY::XBOX + xr * 128 +
                                                                 ((chunk ^ (xr & 7)) << 4)), xf);
                        const float4 c0 = *reinterpret_cast<const float4 *>(cj + 8 * c8);
                        const float4 c1 = *reinterpret_cast<const float4 *>(cj + 8 * c8 + 4);
                        const float cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                        for (int i = 0; i < 8; ++i) a[8 * c8 + i] = fmaf(cw[i], xf[i], a[8 * c8 + i]);
                    }
                }
#pragma unroll
                for (int c8 = 0; c8 < 2; ++c8) {
                    uint4 hi, lo;
                    split8(a + 8 * c8, hi, lo);
                    const uint32_t off = sw128_off(row, acol + 8 * c8, LY::A_BLK);
                    st16(sm + LY::A, off, hi);
                    st16(sm + LY::A_LO, off, lo);
                }
            }
            if constexpr (D == 64) {
#pragma unroll
                for (int c8 = 0; c8 < 2; ++c8) {
                    const int chunk = (col0 >> 3) + c8;
                    unpack8(*reinterpret_cast<const uint4 *>(sm + LY::V + row * 128 + ((chunk ^ (row & 7)) << 4)),
                            r + 8 * c8);
                }
            } else {
                unpack8(vnext[0], r);
                unpack8(vnext[1], r + 8);
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
                tmem_ld16(taddr(tb, 32 * q, slot * 2 * NH + col0), kk);
                tmem_ld16(taddr(tb, 32 * q, slot * 2 * NH + NH + col0), pp);
                tmem_wait_ld();
                fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_free[slot]);
                // global loads after the arrive (an arrive waits for this thread's loads in flight)
                const float bcur = bl;
                if (l + 1 < L && live) bl = p.beta[tok * L + l + 1];
                if constexpr (D != 64)
                    if (l + 1 == L && tw.left > 1) {
                        TileWalk nx = tw;
                        nx.next();
                        load_v(nx.j, nx.b(), nx.h());
                    }
                put(box(), kk, &maps.w, l, h, t0, b);
                gelu_step<RCW>(pp, r, bcur, pp);
                put(box(), pp, &maps.u, l, h, t0, b);
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
bool weight_map(CUtensorMap *m, const void *base, int H, int L, int d, int rows) {
    auto enc = map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)d, (cuuint64_t)L, (cuuint64_t)H};
    const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)d * d * 2, (cuuint64_t)L * d * d * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)rows, 1, 1};
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

template <int D>
cudaError_t launch_producer_ring(const ProducerArgs &a, cudaStream_t s) {
    using LY = RingLayout<D>;
    RingMaps maps;
    if (!act_map(&maps.x, a.x, a.B, a.T, a.H, D, LY::XROWS) || !act_map(&maps.v, a.v, a.B, a.T, a.H, D, PT) ||
        !weight_map(&maps.wk, a.Wk, a.H, a.L, D, LY::NH) || !weight_map(&maps.wp, a.Wp, a.H, a.L, D, LY::NH) ||
        !out_map(&maps.u, a.u, a.B, a.T, a.H, a.L, D) || !out_map(&maps.w, a.w, a.B, a.T, a.H, a.L, D))
        return cudaErrorInvalidValue;
    auto kern = write_producer_ring_kernel<D>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)LY::BYTES);
    if (err != cudaSuccess) return err;
    const long long ntiles = (long long)a.H * a.B * ((a.T + PT - 1) / PT);
    const int pairs = (int)std::min<long long>(ntiles, std::max(1, device_sms() / LY::HALVES));
    launch_probe_mark(s);
    kern<<<pairs * LY::HALVES, LY::THREADS, LY::BYTES, s>>>(a, maps, ntiles);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_write_producer(const ProducerArgs &a, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    return a.d == 128 ? launch_producer_ring<128>(a, s) : launch_producer_ring<64>(a, s);
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
