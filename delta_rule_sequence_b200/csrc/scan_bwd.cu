// scan_bwd.cu -- the backward pass of the scan: gradients of every input of prism_scan_fwd, fp32
// on CUDA cores.
//
// The forward is the token recurrence of PRISM (gist.science explainer, technical summary 2.1 and
// 2.2; banbantang.com PRISM article, section 1(4)):
//   S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + W_t,   o_t = S_t q_t,
//   W_t = beta_t v_t k_t^T (Gated-DeltaNet write) or sum_l u_{t,l} w_{t,l}^T (rank-L write).
// For upstream gradients do_t and dS_T, the gradient G_t of S_t runs backwards from G_T = dS_T:
//   G_t += do_t q_t^T;   dq_t = S_t^T do_t;
//   dalpha_t = <G_t, S_{t-1}> - beta_t (S_{t-1}k_t).(G_t k_t);
//   dbeta_t  = -alpha_t (S_{t-1}k_t).(G_t k_t)  [+ v_t.(G_t k_t)];
//   dk_t     = -alpha_t beta_t (G_t^T S_{t-1}k_t + S_{t-1}^T G_t k_t)  [+ beta_t G_t^T v_t];
//   dv_t = beta_t G_t k_t  |  du_{t,l} = G_t w_{t,l},  dw_{t,l} = G_t^T u_{t,l};
//   G_{t-1} = alpha_t (G_t - beta_t (G_t k_t) k_t^T);   dS0 = G_0.
// Row r of S and of G evolves on its own (the recurrence multiplies S from the right), so the
// value rows are split over CTAs and warps: one warp owns one row (lane j holds columns j, j + 32,
// ...), its dot products are warp reductions, and only dq, dk, dw, dalpha and dbeta sum over rows
// (per token in shared memory across the CTA's warps, then one atomic add per element and CTA).
//
// The backward needs S_{t-1} and S_t at every token, in reverse order.  Each CTA first runs the
// forward recurrence for its rows and writes the state at every 64-token chunk start to the
// workspace; then, chunk by chunk from the last, it recomputes the chunk's states from that
// checkpoint into a per-CTA workspace buffer (and S_{t-1} k_t into shared memory) and walks the
// chunk's tokens backwards.  All arithmetic is fp32 from the exact input values.

#include "common.cuh"

namespace prism {
namespace {

constexpr int BW_NW = 16;              // value rows (warps) per CTA
constexpr int BW_THREADS = 32 * BW_NW;
constexpr int BW_C = 64;               // tokens between checkpoints
constexpr int BW_TS = 8;               // tokens per flush of the cross-row sums

struct BwdArgs {
    int B, H, T, dk, dv, L, nch;
    const void *q, *k, *v, *u, *w, *dO;
    const float *alpha, *beta, *S0, *dS_final;
    float *dq, *dk_out, *dv_out, *dalpha, *dbeta, *du, *dw, *dS0;
    float *ckpt;     // [B, H, nch, dv, dk] state at each chunk start
    float *scratch;  // per CTA: [BW_C + 1][BW_NW][dk] states of the current chunk
};

template <int DK>
struct BwdSmem {
    // cross-row sums of BW_TS tokens: dq, dk, dw (L ranks), dalpha, dbeta; S_{t-1} k_t per warp
    static size_t bytes(int L) {
        return sizeof(float) * ((size_t)(2 + L) * BW_TS * DK + 2 * BW_TS + (size_t)BW_NW * BW_C);
    }
};

template <typename IO, int DK>
__global__ void __launch_bounds__(BW_THREADS) scan_bwd_kernel(BwdArgs p) {
    constexpr int E = DK / 32;  // columns per lane
    extern __shared__ float smem[];
    const int L = p.L;
    float *acc_dq = smem;                      // [BW_TS][DK]
    float *acc_dk = acc_dq + BW_TS * DK;       // [BW_TS][DK]
    float *acc_dw = acc_dk + BW_TS * DK;       // [BW_TS][L][DK]
    float *acc_da = acc_dw + (size_t)BW_TS * L * DK;  // [BW_TS]
    float *acc_db = acc_da + BW_TS;            // [BW_TS]
    float *pk_all = acc_db + BW_TS;            // [BW_NW][BW_C]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = blockIdx.x * BW_NW + warp;   // value row of this warp
    const int h = blockIdx.y, b = blockIdx.z;
    const int H = p.H, T = p.T, dv = p.dv, nch = p.nch;
    const bool gdn = p.u == nullptr;
    const size_t head = (size_t)b * H + h;
    const IO *q = (const IO *)p.q, *k = (const IO *)p.k, *v = (const IO *)p.v;
    const IO *u = (const IO *)p.u, *w = (const IO *)p.w, *dO = (const IO *)p.dO;
    float *pk = pk_all + warp * BW_C;
    const size_t cta = ((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
    float *scr = p.scratch + cta * (size_t)(BW_C + 1) * BW_NW * DK + warp * DK;  // + i * NW * DK

    auto tok = [&](int t) { return ((size_t)b * T + t) * H + h; };  // index of (b, t, h)
    auto load_row = [&](const IO *base, size_t off, float (&x)[E]) {
#pragma unroll
        for (int i = 0; i < E; ++i) x[i] = ld_io<IO>(base, off + lane + 32 * i);
    };
    auto dot = [&](const float (&a)[E], const float (&c)[E]) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < E; ++i) s = fmaf(a[i], c[i], s);
        return warp_sum(s);
    };
    // one forward step of row r at token t; returns S_{t-1} k_t (of this row)
    auto step = [&](float (&s)[E], int t) -> float {
        float kk[E];
        load_row(k, tok(t) * DK, kk);
        const float sk = dot(s, kk);
        const float a = p.alpha[tok(t)], be = p.beta[tok(t)];
#pragma unroll
        for (int i = 0; i < E; ++i) s[i] = a * fmaf(-be * sk, kk[i], s[i]);
        if (gdn) {
            const float bv = be * ld_io<IO>(v, tok(t) * dv + r);
#pragma unroll
            for (int i = 0; i < E; ++i) s[i] = fmaf(bv, kk[i], s[i]);
        } else {
            for (int l = 0; l < L; ++l) {
                float ww[E];
                load_row(w, (tok(t) * L + l) * DK, ww);
                const float ur = ld_io<IO>(u, (tok(t) * L + l) * dv + r);
#pragma unroll
                for (int i = 0; i < E; ++i) s[i] = fmaf(ur, ww[i], s[i]);
            }
        }
        return sk;
    };
    auto store_state = [&](float *dst, const float (&s)[E]) {
#pragma unroll
        for (int i = 0; i < E; ++i) dst[lane + 32 * i] = s[i];
    };
    auto load_state = [&](const float *src, float (&s)[E]) {
#pragma unroll
        for (int i = 0; i < E; ++i) s[i] = src[lane + 32 * i];
    };
    auto ckpt_row = [&](int c) { return p.ckpt + (((head * nch + c) * dv) + r) * DK; };

    // 1. forward over the whole sequence, checkpointing this row at every chunk start
    float s[E];
    if (p.S0) load_state(p.S0 + (head * dv + r) * DK, s);
    else {
#pragma unroll
        for (int i = 0; i < E; ++i) s[i] = 0.f;
    }
    for (int c = 0; c < nch; ++c) {
        store_state(ckpt_row(c), s);
        const int c0 = c * BW_C, n = min(BW_C, T - c0);
        for (int i = 0; i < n; ++i) step(s, c0 + i);
    }

    // 2. backward, chunk by chunk from the last
    float g[E];
    if (p.dS_final) load_state(p.dS_final + (head * dv + r) * DK, g);
    else {
#pragma unroll
        for (int i = 0; i < E; ++i) g[i] = 0.f;
    }
    const int acc_n = (2 + L) * BW_TS * DK + 2 * BW_TS;
    for (int e = tid; e < acc_n; e += BW_THREADS) smem[e] = 0.f;
    __syncthreads();
    for (int c = nch - 1; c >= 0; --c) {
        const int c0 = c * BW_C, n = min(BW_C, T - c0);
        // the chunk's states S_{c0-1+i} (i = 0..n) and S_{t-1} k_t, recomputed from the checkpoint
        load_state(ckpt_row(c), s);
        store_state(scr, s);
        for (int i = 0; i < n; ++i) {
            const float sk = step(s, c0 + i);
            if (lane == 0) pk[i] = sk;
            store_state(scr + (size_t)(i + 1) * BW_NW * DK, s);
        }
        __syncwarp();
        for (int i = n - 1; i >= 0; --i) {
            const int t = c0 + i, slot = i % BW_TS;
            float sp[E], sc[E], kk[E], qq[E];
            load_state(scr + (size_t)i * BW_NW * DK, sp);
            load_state(scr + (size_t)(i + 1) * BW_NW * DK, sc);
            load_row(k, tok(t) * DK, kk);
            load_row(q, tok(t) * DK, qq);
            const float dd = ld_io<IO>(dO, tok(t) * dv + r);
            const float a = p.alpha[tok(t)], be = p.beta[tok(t)];
            const float Pk = pk[i];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                g[e] = fmaf(dd, qq[e], g[e]);
                atomicAdd(&acc_dq[slot * DK + lane + 32 * e], dd * sc[e]);
            }
            const float Gk = dot(g, kk), gs = dot(g, sp);
            float da = gs - be * Pk * Gk, db = -a * Pk * Gk;
            const float ab = a * be;
            float dk_[E];
#pragma unroll
            for (int e = 0; e < E; ++e) dk_[e] = -ab * fmaf(g[e], Pk, sp[e] * Gk);
            if (gdn) {
                const float vr = ld_io<IO>(v, tok(t) * dv + r);
                db = fmaf(vr, Gk, db);
#pragma unroll
                for (int e = 0; e < E; ++e) dk_[e] = fmaf(be * vr, g[e], dk_[e]);
                if (lane == 0) p.dv_out[tok(t) * dv + r] = be * Gk;
            } else {
                for (int l = 0; l < L; ++l) {
                    float ww[E];
                    load_row(w, (tok(t) * L + l) * DK, ww);
                    const float ur = ld_io<IO>(u, (tok(t) * L + l) * dv + r);
                    const float dul = dot(g, ww);
                    if (lane == 0) p.du[(tok(t) * L + l) * dv + r] = dul;
#pragma unroll
                    for (int e = 0; e < E; ++e)
                        atomicAdd(&acc_dw[((size_t)slot * L + l) * DK + lane + 32 * e], ur * g[e]);
                }
            }
#pragma unroll
            for (int e = 0; e < E; ++e) atomicAdd(&acc_dk[slot * DK + lane + 32 * e], dk_[e]);
            if (lane == 0) {
                atomicAdd(&acc_da[slot], da);
                atomicAdd(&acc_db[slot], db);
            }
#pragma unroll
            for (int e = 0; e < E; ++e) g[e] = a * fmaf(-be * Gk, kk[e], g[e]);
            if (slot == 0) {
                // tokens i .. i + m - 1 of the chunk are complete: add this CTA's row sums to the
                // global gradients, then clear the slots
                __syncthreads();
                const int m = min(BW_TS, n - i);
                for (int e = tid; e < m * DK; e += BW_THREADS) {
                    const int sl = e / DK, j = e % DK;
                    const size_t o = tok(t + sl) * DK + j;
                    atomicAdd(&p.dq[o], acc_dq[sl * DK + j]);
                    atomicAdd(&p.dk_out[o], acc_dk[sl * DK + j]);
                    acc_dq[sl * DK + j] = 0.f;
                    acc_dk[sl * DK + j] = 0.f;
                }
                if (!gdn) {
                    for (int e = tid; e < m * L * DK; e += BW_THREADS) {
                        const int sl = e / (L * DK), l = (e / DK) % L, j = e % DK;
                        atomicAdd(&p.dw[(tok(t + sl) * L + l) * DK + j], acc_dw[e]);
                        acc_dw[e] = 0.f;
                    }
                }
                if (tid < m) {
                    atomicAdd(&p.dalpha[tok(t + tid)], acc_da[tid]);
                    atomicAdd(&p.dbeta[tok(t + tid)], acc_db[tid]);
                    acc_da[tid] = 0.f;
                    acc_db[tid] = 0.f;
                }
                __syncthreads();
            }
        }
    }
    if (p.dS0) store_state(p.dS0 + (head * dv + r) * DK, g);
}

template <typename IO, int DK>
cudaError_t launch_bwd_t(const BwdArgs &a, cudaStream_t s) {
    const size_t bytes = BwdSmem<DK>::bytes(a.L);
    auto kern = scan_bwd_kernel<IO, DK>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (err != cudaSuccess) return err;
    dim3 grid(a.dv / BW_NW, a.H, a.B);
    launch_probe_mark(s);
    kern<<<grid, BW_THREADS, bytes, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

// Workspace of the backward after the status block: the chunk-start states of every row, and one
// chunk of states per CTA.
size_t bwd_workspace_bytes(int B, int H, int T, int dk, int dv) {
    const size_t nch = (size_t)((T + BW_C - 1) / BW_C);
    const size_t ctas = (size_t)B * H * (dv / BW_NW);
    return kStatusBytes + sizeof(float) * ((size_t)B * H * nch * dv * dk + ctas * (BW_C + 1) * BW_NW * dk);
}

// The gradients (fp32).  dq, dk, dw, dalpha, dbeta are sums over value rows (atomic adds): they are
// cleared on the stream first.  dv / du and dS0 are written once per element.
cudaError_t launch_scan_bwd(const ScanArgs &f, const void *dO, const float *dS_final, float *dq,
                            float *dk, float *dv, float *dalpha, float *dbeta, float *du, float *dw,
                            float *dS0, void *ws, bool io_f32, cudaStream_t s) {
    const size_t tok = (size_t)f.B * f.T * f.H;
    cudaError_t err;
    if (tok > 0) {
        if ((err = cudaMemsetAsync(dq, 0, tok * f.dk * sizeof(float), s)) != cudaSuccess) return err;
        if ((err = cudaMemsetAsync(dk, 0, tok * f.dk * sizeof(float), s)) != cudaSuccess) return err;
        if ((err = cudaMemsetAsync(dalpha, 0, tok * sizeof(float), s)) != cudaSuccess) return err;
        if ((err = cudaMemsetAsync(dbeta, 0, tok * sizeof(float), s)) != cudaSuccess) return err;
        if (dw && (err = cudaMemsetAsync(dw, 0, tok * f.L * f.dk * sizeof(float), s)) != cudaSuccess)
            return err;
    }
    if (f.T == 0) {  // no tokens: dS0 = dS_final
        if (!dS0) return cudaSuccess;
        const size_t n = (size_t)f.B * f.H * f.dv * f.dk * sizeof(float);
        return dS_final ? cudaMemcpyAsync(dS0, dS_final, n, cudaMemcpyDeviceToDevice, s)
                        : cudaMemsetAsync(dS0, 0, n, s);
    }
    BwdArgs a;
    a.B = f.B; a.H = f.H; a.T = f.T; a.dk = f.dk; a.dv = f.dv; a.L = f.L;
    a.nch = (f.T + BW_C - 1) / BW_C;
    a.q = f.q; a.k = f.k; a.v = f.v; a.u = f.u; a.w = f.w; a.dO = dO;
    a.alpha = f.alpha; a.beta = f.beta; a.S0 = f.S0; a.dS_final = dS_final;
    a.dq = dq; a.dk_out = dk; a.dv_out = dv; a.dalpha = dalpha; a.dbeta = dbeta;
    a.du = du; a.dw = dw; a.dS0 = dS0;
    a.ckpt = (float *)((uint8_t *)ws + kStatusBytes);
    a.scratch = a.ckpt + (size_t)f.B * f.H * a.nch * f.dv * f.dk;
    if (io_f32) {
        switch (f.dk) {
            case 32: return launch_bwd_t<float, 32>(a, s);
            case 64: return launch_bwd_t<float, 64>(a, s);
            case 128: return launch_bwd_t<float, 128>(a, s);
        }
    } else {
        switch (f.dk) {
            case 32: return launch_bwd_t<__nv_bfloat16, 32>(a, s);
            case 64: return launch_bwd_t<__nv_bfloat16, 64>(a, s);
            case 128: return launch_bwd_t<__nv_bfloat16, 128>(a, s);
        }
    }
    return cudaErrorInvalidValue;
}

}  // namespace prism
