// decode.cu -- single-token recurrent step: an HBM-bound rank-(L+1) update of the fp32 state.
//
// For each (b, h) and each state row s_r (length dk), with e_r = s_r.k and p_r = s_r.q:
//   s_r <- alpha s_r - alpha beta e_r k + sum_l u_{l,r} w_l
//   o_r  = alpha p_r - alpha beta e_r (k.q) + sum_l u_{l,r} (w_l.q)
// i.e. S <- alpha S (I - beta k k^T) + sum_l u_l w_l^T and o = S q with the updated S (PRISM,
// gist.science explainer, technical summary 2.1-2.2; streaming inference of "Sequential Parallel
// Duality in Prefix Scannable Models": one state updated per token, since the monoid is
// associative).  The state is read once and written once; everything else is a few KB per head.
//
// Layout: one CTA (8 warps) per head; a warp owns blocks of 8 consecutive rows; a lane holds
// dk/32 consecutive columns (a 16-byte vector at dk = 128).  The state is streamed: it is far
// larger than L2 and touched once per step.
//
// Two variants.  `decode_ring_kernel` (dk = 128, dv = 64 or 128) is persistent, one CTA per SM:
// each head's state and token vectors arrive in one of three shared-memory stages by bulk copies
// (cp.async.bulk) issued three heads ahead, so that the bytes in flight per SM are set by shared
// memory rather than by registers and stay in flight while the current head is updated.
// `decode_kernel` (every other shape) loads 8 rows per warp into registers (evict-first) before
// reducing any of them.

#include "tc.cuh"

namespace prism {
namespace {

constexpr int NT = 256;
constexpr int NW = NT / 32;
constexpr int ROWS_IN_FLIGHT = 8;

template <int N>
struct VecF;
template <> struct VecF<1> { using T = float; };
template <> struct VecF<2> { using T = float2; };
template <> struct VecF<4> { using T = float4; };

template <int N>
__device__ __forceinline__ void vload(const float *p, float (&x)[N]) {
    using V = typename VecF<N>::T;
    V t = __ldcs(reinterpret_cast<const V *>(p));
    const float *f = reinterpret_cast<const float *>(&t);
#pragma unroll
    for (int i = 0; i < N; ++i) x[i] = f[i];
}

template <int N>
__device__ __forceinline__ void vstore(float *p, const float (&x)[N]) {
    using V = typename VecF<N>::T;
    V t;
    float *f = reinterpret_cast<float *>(&t);
#pragma unroll
    for (int i = 0; i < N; ++i) f[i] = x[i];
    __stcs(reinterpret_cast<V *>(p), t);
}

template <int N>
__device__ __forceinline__ void vload_shared(const float *p, float (&x)[N]) {
    using V = typename VecF<N>::T;
    V t = *reinterpret_cast<const V *>(p);
    const float *f = reinterpret_cast<const float *>(&t);
#pragma unroll
    for (int i = 0; i < N; ++i) x[i] = f[i];
}

// Reduce-scatter of 8 per-lane partial sums (rows j = 0..7 of a block) over the warp: afterwards
// every lane holds the full sum of row lane / 4.  Three exchange steps halve the rows a lane keeps
// (offsets 16, 8, 4: 4 + 2 + 1 shuffles), two more finish the sum over the lanes sharing a row.
__device__ __forceinline__ float rows8_reduce_scatter(const float (&x)[ROWS_IN_FLIGHT], int lane) {
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
    float y[4], z[2];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float send = b4 ? x[j] : x[j + 4], keep = b4 ? x[j + 4] : x[j];
        y[j] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const float send = b3 ? y[j] : y[j + 2], keep = b3 ? y[j + 2] : y[j];
        z[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    float r = (b2 ? z[1] : z[0]) + __shfl_xor_sync(0xffffffffu, b2 ? z[0] : z[1], 4);
    r += __shfl_xor_sync(0xffffffffu, r, 2);
    r += __shfl_xor_sync(0xffffffffu, r, 1);
    return r;
}

// Library status word of the decode kernels (a bounded wait that gave up), read and cleared by
// prism_query_device_status.
__device__ uint32_t g_decode_status;

// The per-head prologue shared by both variants: k, q in registers; w_l (or k) and u_{l,r} (or
// beta v_r) in shared memory; k.q; the w_l.q in shared memory.
template <typename IO, int DK, int LW>
struct DecodeHead {
    float kq[DK / 32], qv[DK / 32];
    float kdotq;
};

template <typename IO, int DK, int LW>
__device__ __forceinline__ void decode_prologue(const ScanArgs &p, int head, float (&s_u)[LW][128],
                                                float (&s_w)[LW][DK], float (&s_wq)[LW],
                                                DecodeHead<IO, DK, LW> &hd) {
    constexpr int PER = DK / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int dv = p.dv, L = p.L;
    const bool gdn = (p.u == nullptr);
    const IO *q = (const IO *)p.q, *k = (const IO *)p.k, *v = (const IO *)p.v;
    const IO *u = (const IO *)p.u, *w = (const IO *)p.w;
    const float be = p.beta[head];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        size_t idx = (size_t)head * DK + lane * PER + i;
        hd.kq[i] = ld_io(k, idx);
        hd.qv[i] = ld_io(q, idx);
    }
    for (int e = threadIdx.x; e < LW * DK; e += NT) {
        int l = e / DK, j = e % DK;
        s_w[l][j] = gdn ? ld_io(k, (size_t)head * DK + j) : ld_io(w, ((size_t)head * L + l) * DK + j);
    }
    for (int e = threadIdx.x; e < LW * dv; e += NT) {
        int l = e / dv, r = e % dv;
        s_u[l][r] = gdn ? be * ld_io(v, (size_t)head * dv + r) : ld_io(u, ((size_t)head * L + l) * dv + r);
    }
    float kdotq = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) kdotq = fmaf(hd.kq[i], hd.qv[i], kdotq);
    hd.kdotq = warp_sum(kdotq);
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int l = 0; l < LW; ++l) {
            float t = 0.f;
#pragma unroll
            for (int i = 0; i < PER; ++i) t = fmaf(s_w[l][lane * PER + i], hd.qv[i], t);
            t = warp_sum(t);
            if (lane == 0) s_wq[l] = t;
        }
    }
    __syncthreads();
}

// One block of 8 rows r0 .. r0 + 7 held in registers (s[j] = row r0 + j, this lane's columns):
// the output o_r and the new rows, stored with evict-first stores.
template <typename IO, int DK, int LW>
__device__ __forceinline__ void decode_rows8(const ScanArgs &p, int head, int r0,
                                             float (&s)[ROWS_IN_FLIGHT][DK / 32],
                                             const float (&s_u)[LW][128], const float (&s_w)[LW][DK],
                                             const float (&s_wq)[LW], const DecodeHead<IO, DK, LW> &hd) {
    constexpr int PER = DK / 32;
    const int lane = threadIdx.x & 31;
    const float a = p.alpha[head];
    const float ab = a * p.beta[head];
    IO *o = (IO *)p.o + (size_t)head * p.dv;
    float *S = p.S_final + (size_t)head * p.dv * DK;
    const int my_row = lane >> 2;  // the row of the block whose sums this lane ends up holding
    // e_r = s_r . k and p_r = s_r . q for the 8 rows: per-lane partials, then one butterfly
    float ep[ROWS_IN_FLIGHT], pp[ROWS_IN_FLIGHT];
#pragma unroll
    for (int j = 0; j < ROWS_IN_FLIGHT; ++j) {
        float e = 0.f, pq = 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            e = fmaf(s[j][i], hd.kq[i], e);
            pq = fmaf(s[j][i], hd.qv[i], pq);
        }
        ep[j] = e;
        pp[j] = pq;
    }
    const float e_mine = rows8_reduce_scatter(ep, lane);
    const float p_mine = rows8_reduce_scatter(pp, lane);
    // o_r = alpha p_r - alpha beta e_r (k.q) + sum_l u_{l,r} (w_l.q), by lane 4 r
    if ((lane & 3) == 0) {
        const int r = r0 + my_row;
        float outv = a * p_mine - ab * e_mine * hd.kdotq;
#pragma unroll
        for (int l = 0; l < LW; ++l) outv = fmaf(s_u[l][r], s_wq[l], outv);
        st_io(o, r, outv);
    }
    // s_r <- alpha s_r - alpha beta e_r k + sum_l u_{l,r} w_l
#pragma unroll
    for (int j = 0; j < ROWS_IN_FLIGHT; ++j) {
        const float ej = __shfl_sync(0xffffffffu, e_mine, 4 * j);
#pragma unroll
        for (int i = 0; i < PER; ++i) s[j][i] = fmaf(a, s[j][i], -ab * ej * hd.kq[i]);
    }
#pragma unroll
    for (int l = 0; l < LW; ++l) {
        float wv[PER];
        vload_shared<PER>(&s_w[l][lane * PER], wv);
        const float4 u0 = *reinterpret_cast<const float4 *>(&s_u[l][r0]);
        const float4 u1 = *reinterpret_cast<const float4 *>(&s_u[l][r0 + 4]);
        const float uu[ROWS_IN_FLIGHT] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int j = 0; j < ROWS_IN_FLIGHT; ++j) {
#pragma unroll
            for (int i = 0; i < PER; ++i) s[j][i] = fmaf(uu[j], wv[i], s[j][i]);
        }
    }
#pragma unroll
    for (int j = 0; j < ROWS_IN_FLIGHT; ++j) vstore<PER>(S + (size_t)(r0 + j) * DK + lane * PER, s[j]);
}

// dk = 128, dv = DV in {64, 128}: a persistent CTA per SM walks the heads blockIdx.x,
// blockIdx.x + gridDim.x, ...  Each head's state and token vectors (k, q, and u, w or v) arrive in
// one of NSTAGE shared-memory stages by bulk copies issued NSTAGE heads ahead, so that while one
// head is updated the next ones are already in flight; warp w updates rows [w DV/8, (w+1) DV/8)
// in blocks of 8 and stores them with evict-first stores.
constexpr int kDecodeStages = 3;

template <typename IO, int DV, int LW>
struct RingLayout {
    static constexpr int DK = 128;
    static constexpr uint32_t S = 0;                                 // fp32 [DV][DK]
    static constexpr uint32_t K = S + DV * DK * 4;                   // io [DK]
    static constexpr uint32_t Q = K + DK * sizeof(IO);               // io [DK]
    static constexpr uint32_t U = Q + DK * sizeof(IO);               // io [LW][DV] (or v [DV])
    static constexpr uint32_t W = U + LW * DV * sizeof(IO);          // io [LW][DK] (rank L)
    static constexpr uint32_t STAGE = W + LW * DK * sizeof(IO);
    static constexpr uint32_t BYTES = kDecodeStages * STAGE;
    static_assert(STAGE % 16 == 0 && (DK * sizeof(IO)) % 16 == 0, "bulk copies move 16-byte units");
};

template <typename IO, int DV, int LW>
__global__ void __launch_bounds__(NT, 1) decode_ring_kernel(ScanArgs p, int nheads) {
    using LY = RingLayout<IO, DV, LW>;
    constexpr int DK = 128, PER = DK / 32;
    constexpr int RW = DV / NW;  // rows per warp
    static_assert(RW % ROWS_IN_FLIGHT == 0, "a warp's rows come in blocks of 8");
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t full[kDecodeStages];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool gdn = (p.u == nullptr);
    const int L = p.L;
    const IO *qg = (const IO *)p.q, *kg = (const IO *)p.k, *vg = (const IO *)p.v;
    const IO *ug = (const IO *)p.u, *wg = (const IO *)p.w;
    // the give-up test: the copies are not issued and the waits run out after a short limit
    const bool stall = (p.flags & kStallDecode) != 0;
    const uint32_t lim = stall ? kStallTestPolls : kWaitPolls;

    auto issue = [&](int st, int head) {  // thread 0: one head into stage st
        uint8_t *dst = smem + st * LY::STAGE;
        const uint32_t vec = gdn ? DV * sizeof(IO) : LW * (DV + DK) * sizeof(IO);
        tc::mbar_expect_tx(&full[st], DV * DK * 4 + 2 * DK * sizeof(IO) + vec);
        tc::bulk_g2s(dst + LY::S, p.S_final + (size_t)head * DV * DK, DV * DK * 4, &full[st]);
        tc::bulk_g2s(dst + LY::K, kg + (size_t)head * DK, DK * sizeof(IO), &full[st]);
        tc::bulk_g2s(dst + LY::Q, qg + (size_t)head * DK, DK * sizeof(IO), &full[st]);
        if (gdn) {
            tc::bulk_g2s(dst + LY::U, vg + (size_t)head * DV, DV * sizeof(IO), &full[st]);
        } else {
            tc::bulk_g2s(dst + LY::U, ug + (size_t)head * LW * DV, LW * DV * sizeof(IO), &full[st]);
            tc::bulk_g2s(dst + LY::W, wg + (size_t)head * LW * DK, LW * DK * sizeof(IO), &full[st]);
        }
    };
    const int first = blockIdx.x, step = gridDim.x;
    const int mine = first < nheads ? (nheads - 1 - first) / step + 1 : 0;  // heads of this CTA
    if (threadIdx.x == 0) {
        for (int i = 0; i < kDecodeStages; ++i) tc::mbar_init(&full[i], 1);
        tc::mbar_fence_init();
        if (!stall)
            for (int i = 0; i < kDecodeStages && i < mine; ++i) issue(i, first + i * step);
    }
    __syncthreads();
    int done = 0;  // heads consumed
    for (int i = 0; i < mine; ++i) {
        const int st = i % kDecodeStages, head = first + i * step;
        const bool landed = tc::mbar_wait(&full[st], (i / kDecodeStages) & 1, &g_decode_status, lim);
        if (__syncthreads_or(!landed)) break;
        const uint8_t *stg = smem + st * LY::STAGE;
        const float *sS = reinterpret_cast<const float *>(stg + LY::S);
        const IO *sk = reinterpret_cast<const IO *>(stg + LY::K);
        const IO *sq = reinterpret_cast<const IO *>(stg + LY::Q);
        const IO *su = reinterpret_cast<const IO *>(stg + LY::U);
        const IO *sw = gdn ? sk : reinterpret_cast<const IO *>(stg + LY::W);
        const float a = p.alpha[head], be = p.beta[head], ab = a * be;
        float kq[PER], qv[PER];
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            kq[e] = ld_io(sk, lane * PER + e);
            qv[e] = ld_io(sq, lane * PER + e);
        }
        float kdotq = 0.f;
#pragma unroll
        for (int e = 0; e < PER; ++e) kdotq = fmaf(kq[e], qv[e], kdotq);
        kdotq = warp_sum(kdotq);
        float wq[LW];  // w_l . q (every warp computes its own copy)
#pragma unroll
        for (int l = 0; l < LW; ++l) {
            float t = 0.f;
#pragma unroll
            for (int e = 0; e < PER; ++e) t = fmaf(ld_io(sw, (gdn ? 0 : l * DK) + lane * PER + e), qv[e], t);
            wq[l] = warp_sum(t);
        }
        IO *o = (IO *)p.o + (size_t)head * DV;
        float *S = p.S_final + (size_t)head * DV * DK;
        const int my_row = lane >> 2;
        for (int rb = 0; rb < RW; rb += ROWS_IN_FLIGHT) {
            const int r0 = warp * RW + rb;
            float s[ROWS_IN_FLIGHT][PER];
#pragma unroll
            for (int j = 0; j < ROWS_IN_FLIGHT; ++j)
                vload_shared<PER>(sS + (size_t)(r0 + j) * DK + lane * PER, s[j]);
            float ep[ROWS_IN_FLIGHT], pp[ROWS_IN_FLIGHT];
#pragma unroll
            for (int j = 0; j < ROWS_IN_FLIGHT; ++j) {
                float e = 0.f, pq = 0.f;
#pragma unroll
                for (int c = 0; c < PER; ++c) {
                    e = fmaf(s[j][c], kq[c], e);
                    pq = fmaf(s[j][c], qv[c], pq);
                }
                ep[j] = e;
                pp[j] = pq;
            }
            const float e_mine = rows8_reduce_scatter(ep, lane);
            const float p_mine = rows8_reduce_scatter(pp, lane);
            // u_{l,r} of the 8 rows (beta v_r on the Gated-DeltaNet write)
            float uu[LW][ROWS_IN_FLIGHT];
#pragma unroll
            for (int l = 0; l < LW; ++l)
#pragma unroll
                for (int j = 0; j < ROWS_IN_FLIGHT; ++j)
                    uu[l][j] = gdn ? be * ld_io(su, r0 + j) : ld_io(su, l * DV + r0 + j);
            if ((lane & 3) == 0) {
                const int r = r0 + my_row;
                float outv = a * p_mine - ab * e_mine * kdotq;
#pragma unroll
                for (int l = 0; l < LW; ++l)
                    outv = fmaf(gdn ? be * ld_io(su, r) : ld_io(su, l * DV + r), wq[l], outv);
                st_io(o, r, outv);
            }
#pragma unroll
            for (int j = 0; j < ROWS_IN_FLIGHT; ++j) {
                const float ej = __shfl_sync(0xffffffffu, e_mine, 4 * j);
#pragma unroll
                for (int c = 0; c < PER; ++c) s[j][c] = fmaf(a, s[j][c], -ab * ej * kq[c]);
            }
#pragma unroll
            for (int l = 0; l < LW; ++l) {
                float wv[PER];
#pragma unroll
                for (int c = 0; c < PER; ++c) wv[c] = ld_io(sw, (gdn ? 0 : l * DK) + lane * PER + c);
#pragma unroll
                for (int j = 0; j < ROWS_IN_FLIGHT; ++j)
#pragma unroll
                    for (int c = 0; c < PER; ++c) s[j][c] = fmaf(uu[l][j], wv[c], s[j][c]);
            }
#pragma unroll
            for (int j = 0; j < ROWS_IN_FLIGHT; ++j) vstore<PER>(S + (size_t)(r0 + j) * DK + lane * PER, s[j]);
        }
        ++done;
        __syncthreads();  // every warp is done with this stage: it takes the head NSTAGE ahead
        if (threadIdx.x == 0 && !stall && i + kDecodeStages < mine)
            issue(st, first + (i + kDecodeStages) * step);
    }
    // after a wait that gave up, the copies still in flight land before the CTA exits (bounded)
    if (threadIdx.x == 0 && !stall) {
        for (int i = done; i < mine && i < done + kDecodeStages; ++i)
            tc::mbar_wait(&full[i % kDecodeStages], (i / kDecodeStages) & 1, nullptr);
    }
}

// LW = number of write terms (L, or 1 for the Gated-DeltaNet write beta v k^T).
template <typename IO, int DK, int LW>
__global__ void __launch_bounds__(NT, 3) decode_kernel(ScanArgs p) {
    constexpr int PER = DK / 32;  // columns per lane
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int head = blockIdx.x;  // b * H + h
    const int dv = p.dv;
    __shared__ __align__(16) float s_u[LW][128];  // u_{l,r} (or beta v_r)
    __shared__ __align__(16) float s_w[LW][DK];   // w_l (or k)
    __shared__ float s_wq[LW];

    // Issue the loads of this warp's first block of state rows before the per-head prologue,
    // so that their latency overlaps the prologue's.
    const float *S = p.S_final + (size_t)head * dv * DK;  // in place
    float s[ROWS_IN_FLIGHT][PER];
    int r0 = warp * ROWS_IN_FLIGHT;
    if (r0 < dv) {
#pragma unroll
        for (int j = 0; j < ROWS_IN_FLIGHT; ++j)
            vload<PER>(S + (size_t)(r0 + j) * DK + lane * PER, s[j]);
    }
    DecodeHead<IO, DK, LW> hd;
    decode_prologue<IO, DK, LW>(p, head, s_u, s_w, s_wq, hd);
    for (; r0 < dv; r0 += NW * ROWS_IN_FLIGHT) {
        if (r0 != warp * ROWS_IN_FLIGHT) {
#pragma unroll
            for (int j = 0; j < ROWS_IN_FLIGHT; ++j)
                vload<PER>(S + (size_t)(r0 + j) * DK + lane * PER, s[j]);
        }
        decode_rows8<IO, DK, LW>(p, head, r0, s, s_u, s_w, s_wq, hd);
    }
}

template <typename IO, int DK, int LW>
cudaError_t launch_decode_l(const ScanArgs &a, cudaStream_t s) {
    if constexpr (DK == 128) {
        if (a.dv == 128 || a.dv == 64) {
            auto kern = a.dv == 128 ? decode_ring_kernel<IO, 128, LW> : decode_ring_kernel<IO, 64, LW>;
            const int bytes = a.dv == 128 ? (int)RingLayout<IO, 128, LW>::BYTES : (int)RingLayout<IO, 64, LW>::BYTES;
            cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
            if (err != cudaSuccess) return err;
            int dev = 0, sms = 148;
            if (cudaGetDevice(&dev) == cudaSuccess)
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            const int heads = a.B * a.H;
            launch_probe_mark(s);
            kern<<<heads < sms ? heads : sms, NT, bytes, s>>>(a, heads);
            return cudaGetLastError();
        }
    }
    launch_probe_mark(s);
    decode_kernel<IO, DK, LW><<<a.B * a.H, NT, 0, s>>>(a);
    return cudaGetLastError();
}

template <typename IO, int DK>
cudaError_t launch_decode_dk(const ScanArgs &a, cudaStream_t s) {
    const int lw = (a.u == nullptr) ? 1 : a.L;
    switch (lw) {
        case 1: return launch_decode_l<IO, DK, 1>(a, s);
        case 2: return launch_decode_l<IO, DK, 2>(a, s);
        case 3: return launch_decode_l<IO, DK, 3>(a, s);
        case 4: return launch_decode_l<IO, DK, 4>(a, s);
        case 5: return launch_decode_l<IO, DK, 5>(a, s);
        case 6: return launch_decode_l<IO, DK, 6>(a, s);
        case 7: return launch_decode_l<IO, DK, 7>(a, s);
        case 8: return launch_decode_l<IO, DK, 8>(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

// Entry used by the C ABI.  a.S_final is the in-place state.  Requires dv <= 128, dv a multiple
// of 64 or dv = 32 (rows come in blocks of 8 per warp), L <= 8 (checked by the caller).
cudaError_t launch_decode(const ScanArgs &a, bool io_f32, cudaStream_t s) {
    if (io_f32) {
        switch (a.dk) {
            case 32: return launch_decode_dk<float, 32>(a, s);
            case 64: return launch_decode_dk<float, 64>(a, s);
            case 128: return launch_decode_dk<float, 128>(a, s);
        }
    } else {
        switch (a.dk) {
            case 32: return launch_decode_dk<__nv_bfloat16, 32>(a, s);
            case 64: return launch_decode_dk<__nv_bfloat16, 64>(a, s);
            case 128: return launch_decode_dk<__nv_bfloat16, 128>(a, s);
        }
    }
    return cudaErrorInvalidValue;
}

// Read and clear the decode kernels' status word (PRISM_ERR_TIMEOUT if a bulk copy's wait gave up).
cudaError_t decode_status(uint32_t *out) {
    uint32_t word = 0;
    cudaError_t err = cudaMemcpyFromSymbol(&word, g_decode_status, sizeof word);
    if (err != cudaSuccess) return err;
    if (word != 0) {
        const uint32_t zero = 0;
        if ((err = cudaMemcpyToSymbol(g_decode_status, &zero, sizeof zero)) != cudaSuccess) return err;
    }
    *out = word;
    return cudaSuccess;
}

}  // namespace prism
