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
// dk/32 consecutive columns (a 16-byte vector at dk = 128).  All 8 rows of a block are loaded
// before any is reduced so that every SM keeps enough bytes in flight to saturate HBM.  The state
// is streamed (evict-first loads and stores): it is far larger than L2 and touched once per step.

#include "common.cuh"

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

// LW = number of write terms (L, or 1 for the Gated-DeltaNet write beta v k^T).
template <typename IO, int DK, int LW>
__global__ void __launch_bounds__(NT, 3) decode_kernel(ScanArgs p) {
    constexpr int PER = DK / 32;  // columns per lane
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int head = blockIdx.x;  // b * H + h
    const int dv = p.dv, L = p.L;
    const bool gdn = (p.u == nullptr);
    const IO *q = (const IO *)p.q, *k = (const IO *)p.k, *v = (const IO *)p.v;
    const IO *u = (const IO *)p.u, *w = (const IO *)p.w;

    __shared__ __align__(16) float s_u[LW][128];  // u_{l,r} (or beta v_r)
    __shared__ __align__(16) float s_w[LW][DK];   // w_l (or k)
    __shared__ float s_wq[LW];

    // Issue the loads of this warp's first block of state rows before the per-head prologue,
    // so that their latency overlaps the prologue's.
    float *S = p.S_final + (size_t)head * dv * DK;  // in place
    float s[ROWS_IN_FLIGHT][PER];
    int r0 = warp * ROWS_IN_FLIGHT;
    if (r0 < dv) {
#pragma unroll
        for (int j = 0; j < ROWS_IN_FLIGHT; ++j)
            vload<PER>(S + (size_t)(r0 + j) * DK + lane * PER, s[j]);
    }

    const float a = p.alpha[head];
    const float be = p.beta[head];
    float kq[PER], qv[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        size_t idx = (size_t)head * DK + lane * PER + i;
        kq[i] = ld_io(k, idx);
        qv[i] = ld_io(q, idx);
    }
    for (int e = threadIdx.x; e < LW * DK; e += NT) {
        int l = e / DK, j = e % DK;
        s_w[l][j] = gdn ? ld_io(k, (size_t)head * DK + j)
                        : ld_io(w, ((size_t)head * L + l) * DK + j);
    }
    for (int e = threadIdx.x; e < LW * dv; e += NT) {
        int l = e / dv, r = e % dv;
        s_u[l][r] = gdn ? be * ld_io(v, (size_t)head * dv + r)
                        : ld_io(u, ((size_t)head * L + l) * dv + r);
    }
    // k.q in every warp; warp 0 publishes the w_l.q
    float kdotq = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) kdotq = fmaf(kq[i], qv[i], kdotq);
    kdotq = warp_sum(kdotq);
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int l = 0; l < LW; ++l) {
            float t = 0.f;
#pragma unroll
            for (int i = 0; i < PER; ++i) t = fmaf(s_w[l][lane * PER + i], qv[i], t);
            t = warp_sum(t);
            if (lane == 0) s_wq[l] = t;
        }
    }
    __syncthreads();

    IO *o = (IO *)p.o + (size_t)head * dv;
    const float ab = a * be;
    const int my_row = lane >> 2;  // the row of the block whose sums this lane ends up holding

    for (; r0 < dv; r0 += NW * ROWS_IN_FLIGHT) {
        if (r0 != warp * ROWS_IN_FLIGHT) {
#pragma unroll
            for (int j = 0; j < ROWS_IN_FLIGHT; ++j)
                vload<PER>(S + (size_t)(r0 + j) * DK + lane * PER, s[j]);
        }
        // e_r = s_r . k and p_r = s_r . q for the 8 rows: per-lane partials, then one butterfly
        float ep[ROWS_IN_FLIGHT], pp[ROWS_IN_FLIGHT];
#pragma unroll
        for (int j = 0; j < ROWS_IN_FLIGHT; ++j) {
            float e = 0.f, pq = 0.f;
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                e = fmaf(s[j][i], kq[i], e);
                pq = fmaf(s[j][i], qv[i], pq);
            }
            ep[j] = e;
            pp[j] = pq;
        }
        const float e_mine = rows8_reduce_scatter(ep, lane);
        const float p_mine = rows8_reduce_scatter(pp, lane);
        // o_r = alpha p_r - alpha beta e_r (k.q) + sum_l u_{l,r} (w_l.q), by lane 4 r
        if ((lane & 3) == 0) {
            const int r = r0 + my_row;
            float outv = a * p_mine - ab * e_mine * kdotq;
#pragma unroll
            for (int l = 0; l < LW; ++l) outv = fmaf(s_u[l][r], s_wq[l], outv);
            st_io(o, r, outv);
        }
        // s_r <- alpha s_r - alpha beta e_r k + sum_l u_{l,r} w_l
#pragma unroll
        for (int j = 0; j < ROWS_IN_FLIGHT; ++j) {
            const float ej = __shfl_sync(0xffffffffu, e_mine, 4 * j);
#pragma unroll
            for (int i = 0; i < PER; ++i) s[j][i] = fmaf(a, s[j][i], -ab * ej * kq[i]);
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
}

template <typename IO, int DK, int LW>
cudaError_t launch_decode_l(const ScanArgs &a, cudaStream_t s) {
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

// The decode kernel has no waits: its status is always PRISM_OK.
cudaError_t decode_status(uint32_t *out) {
    *out = PRISM_OK;
    return cudaSuccess;
}

}  // namespace prism
