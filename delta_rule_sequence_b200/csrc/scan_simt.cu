// scan_simt.cu -- fp32 CUDA-core evaluation of the chunked scan (the fp32-I/O path).
//
// One CTA owns one (batch, head, slice of BV value rows) sequence and walks its chunks in order,
// holding the fp32 state slice in shared memory.  Rows of the state evolve independently (each
// row r only ever meets row r of S0 and of u), so value-row slices need no communication.
//
// Per sub-chunk of CS tokens (the chunk form of "Sequential Parallel Duality in Prefix Scannable
// Models", method overview: chunk, encode, scan; exact under any chunking because the affine
// elements compose associatively), with entry state S and g_t = sum_{r<=t} log alpha_r:
//   A_{t,i}  = beta_t e^{g_t-g_i} k_t.k_i (i<t)       Mqk_{t,i} = e^{g_t-g_i} q_t.k_i (i<=t)
//   R        = diag(beta e^g) K S^T + P U~            P_{t,(i,l)} = beta_t e^{g_t-g_i} k_t.w_{i,l}
//   X        = (I + A)^{-1} R      (forward substitution; x_t = alpha_t beta_t S_{t-1} k_t)
//   O        = diag(e^g) Q S^T - Mqk X + Mqw U~       Mqw_{t,(i,l)} = e^{g_t-g_i} q_t.w_{i,l}
//   S'       = e^{g_n} S - X^T D K + U~^T D W~        D_i = e^{g_n - g_i}
// which is the token recurrence S_t = alpha_t S_{t-1}(I - beta_t k_t k_t^T) + sum_l u w^T
// (PRISM, gist.science explainer, technical summary 2.1-2.2) unrolled over the sub-chunk.
// All arithmetic is fp32; the sub-chunk is 32 tokens whatever the requested chunk length.

#include "common.cuh"

namespace prism {
namespace {

constexpr int CS = 32;        // sub-chunk length (one warp lane per token)
constexpr int BV = 32;        // value rows per CTA
constexpr int NT = 256;       // threads per CTA

template <int DK>
struct SimtSmem {
    static constexpr int KS = DK + 1;   // padded row stride of K, Q, W, S
    static constexpr int XS = BV + 1;   // padded row stride of U, R, O
    static constexpr int GS = CS + 1;   // padded row stride of the CS x CS matrices
    static constexpr int floats = BV * KS + 3 * CS * KS + 3 * CS * XS + 4 * CS * GS + 3 * CS;
    static constexpr size_t bytes = sizeof(float) * floats;
};

template <typename IO, int DK>
__global__ void __launch_bounds__(NT) scan_simt_kernel(ScanArgs p) {
    using SM = SimtSmem<DK>;
    constexpr int KS = SM::KS, XS = SM::XS, GS = SM::GS;
    extern __shared__ float smem[];
    float *sS = smem;               // BV x KS   state slice (row v, column j)
    float *sK = sS + BV * KS;       // CS x KS
    float *sQ = sK + CS * KS;       // CS x KS
    float *sW = sQ + CS * KS;       // CS x KS   w_l rows (general write)
    float *sU = sW + CS * KS;       // CS x XS   u_l slice (or beta v)
    float *sR = sU + CS * XS;       // CS x XS   right-hand side, then X
    float *sO = sR + CS * XS;       // CS x XS   output accumulator
    float *sA = sO + CS * XS;       // CS x GS   A (strictly lower)
    float *sM = sA + CS * GS;       // CS x GS   Mqk (lower incl. diagonal)
    float *sKW = sM + CS * GS;      // CS x GS   masked k.w
    float *sQW = sKW + CS * GS;     // CS x GS   masked q.w
    float *sG = sQW + CS * GS;      // CS        g_t
    float *sB = sG + CS;            // CS        beta_t
    float *sD = sB + CS;            // CS        D_i = e^{g_n - g_i} (0 on padding)

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int v0 = blockIdx.x * BV, h = blockIdx.y, b = blockIdx.z;
    const int H = p.H, T = p.T, dv = p.dv, L = p.L;
    const bool gdn = (p.u == nullptr);
    const int nrows = min(BV, dv - v0);  // dv is a multiple of 32, so nrows == BV
    const IO *q = (const IO *)p.q, *k = (const IO *)p.k, *v = (const IO *)p.v;
    const IO *u = (const IO *)p.u, *w = (const IO *)p.w;
    IO *o = (IO *)p.o;
    const size_t head = (size_t)b * H + h;

    for (int e = tid; e < BV * DK; e += NT) {
        int r = e / DK, j = e % DK;
        float s = 0.f;
        if (p.flags & kS0Identity) s = (v0 + r == j) ? 1.f : 0.f;
        else if (p.S0 && r < nrows) s = p.S0[(head * dv + v0 + r) * DK + j];
        sS[r * KS + j] = s;
    }

    for (int c0 = 0; c0 < T; c0 += CS) {
        const int n = min(CS, T - c0);
        // gates: g = inclusive prefix sum of log alpha; padding tokens are identities
        if (warp == 0) {
            const size_t bth = ((size_t)b * T + c0 + lane) * H + h;
            float la = lane < n ? logf(p.alpha[bth]) : 0.f;
            float be = lane < n ? p.beta[bth] : 0.f;
            sG[lane] = warp_inclusive_scan(la, lane);
            sB[lane] = be;
        }
        for (int e = tid; e < CS * DK; e += NT) {
            int t = e / DK, j = e % DK;
            float kv = 0.f, qv = 0.f;
            if (t < n) {
                size_t idx = (((size_t)b * T + c0 + t) * H + h) * DK + j;
                kv = ld_io(k, idx);
                qv = ld_io(q, idx);
            }
            sK[t * KS + j] = kv;
            sQ[t * KS + j] = qv;
        }
        __syncthreads();

        const float gn = sG[CS - 1];  // log-decay of the whole sub-chunk (padding adds 0)
        if (tid < CS) sD[tid] = tid < n ? expf(gn - sG[tid]) : 0.f;

        // A and Mqk
        for (int e = tid; e < CS * CS; e += NT) {
            int t = e / CS, i = e % CS;
            float dkk = 0.f, dqk = 0.f;
            if (i <= t) {
#pragma unroll 8
                for (int j = 0; j < DK; ++j) {
                    float ki = sK[i * KS + j];
                    dkk = fmaf(sK[t * KS + j], ki, dkk);
                    dqk = fmaf(sQ[t * KS + j], ki, dqk);
                }
            }
            float gam = (i <= t) ? expf(sG[t] - sG[i]) : 0.f;
            sA[t * GS + i] = (i < t) ? sB[t] * gam * dkk : 0.f;
            sM[t * GS + i] = gam * dqk;
        }
        // state terms: R = diag(beta e^g) K S^T, O = diag(e^g) Q S^T
        for (int e = tid; e < CS * BV; e += NT) {
            int t = e / BV, r = e % BV;
            float rk = 0.f, rq = 0.f;
#pragma unroll 8
            for (int j = 0; j < DK; ++j) {
                float s = sS[r * KS + j];
                rk = fmaf(sK[t * KS + j], s, rk);
                rq = fmaf(sQ[t * KS + j], s, rq);
            }
            float gt = expf(sG[t]);
            sR[t * XS + r] = sB[t] * gt * rk;
            sO[t * XS + r] = gt * rq;
        }
        __syncthreads();
        {
            const float gdec = expf(gn);
            for (int e = tid; e < BV * DK; e += NT) sS[(e / DK) * KS + e % DK] *= gdec;
        }

        // rank-L write terms (the Gated-DeltaNet write is u = beta v, w = k, L = 1)
        const int Lw = (p.flags & kNoWrite) ? 0 : L;
        for (int l = 0; l < Lw; ++l) {
            const float *Wl = gdn ? sK : sW;
            for (int e = tid; e < CS * XS; e += NT) {
                int i = e / XS, r = e % XS;
                float uv = 0.f;
                if (i < n && r < BV) {
                    size_t bth = ((size_t)b * T + c0 + i) * H + h;
                    uv = gdn ? sB[i] * ld_io(v, bth * dv + v0 + r)
                             : ld_io(u, (bth * L + l) * dv + v0 + r);
                }
                sU[i * XS + r] = uv;
            }
            if (!gdn) {
                for (int e = tid; e < CS * DK; e += NT) {
                    int i = e / DK, j = e % DK;
                    float wv = 0.f;
                    if (i < n) {
                        size_t bth = ((size_t)b * T + c0 + i) * H + h;
                        wv = ld_io(w, (bth * L + l) * DK + j);
                    }
                    sW[i * KS + j] = wv;
                }
            }
            __syncthreads();
            for (int e = tid; e < CS * CS; e += NT) {
                int t = e / CS, i = e % CS;
                float dkw = 0.f, dqw = 0.f;
                if (i <= t) {
#pragma unroll 8
                    for (int j = 0; j < DK; ++j) {
                        float wi = Wl[i * KS + j];
                        dkw = fmaf(sK[t * KS + j], wi, dkw);
                        dqw = fmaf(sQ[t * KS + j], wi, dqw);
                    }
                }
                float gam = (i <= t) ? expf(sG[t] - sG[i]) : 0.f;
                sKW[t * GS + i] = (i < t) ? sB[t] * gam * dkw : 0.f;
                sQW[t * GS + i] = gam * dqw;
            }
            __syncthreads();
            for (int e = tid; e < CS * BV; e += NT) {
                int t = e / BV, r = e % BV;
                float ar = 0.f, ao = 0.f;
                for (int i = 0; i <= t; ++i) {
                    float uv = sU[i * XS + r];
                    ar = fmaf(sKW[t * GS + i], uv, ar);
                    ao = fmaf(sQW[t * GS + i], uv, ao);
                }
                sR[t * XS + r] += ar;
                sO[t * XS + r] += ao;
            }
            for (int e = tid; e < BV * DK; e += NT) {
                int r = e / DK, j = e % DK;
                float acc = 0.f;
                for (int i = 0; i < n; ++i) acc = fmaf(sD[i] * sU[i * XS + r], Wl[i * KS + j], acc);
                sS[r * KS + j] += acc;
            }
            __syncthreads();
        }

        // X = (I + A)^{-1} R by forward substitution, one lane per value column
        if (warp == 0) {
            const int r = lane;
            for (int t = 1; t < n; ++t) {
                float x = sR[t * XS + r];
                for (int i = 0; i < t; ++i) x = fmaf(-sA[t * GS + i], sR[i * XS + r], x);
                sR[t * XS + r] = x;
            }
        }
        __syncthreads();

        // O -= Mqk X ; store o
        for (int e = tid; e < CS * BV; e += NT) {
            int t = e / BV, r = e % BV;
            if (t < n && !(p.flags & kNoOutput)) {
                float acc = sO[t * XS + r];
                for (int i = 0; i <= t; ++i) acc = fmaf(-sM[t * GS + i], sR[i * XS + r], acc);
                size_t bth = ((size_t)b * T + c0 + t) * H + h;
                st_io(o, bth * dv + v0 + r, acc);
            }
        }
        // S -= X^T D K
        for (int e = tid; e < BV * DK; e += NT) {
            int r = e / DK, j = e % DK;
            float acc = 0.f;
            for (int i = 0; i < n; ++i) acc = fmaf(sD[i] * sR[i * XS + r], sK[i * KS + j], acc);
            sS[r * KS + j] -= acc;
        }
        __syncthreads();
    }

    if (p.S_final) {
        for (int e = tid; e < BV * DK; e += NT) {
            int r = e / DK, j = e % DK;
            if (r < nrows) p.S_final[(head * dv + v0 + r) * DK + j] = sS[r * KS + j];
        }
    }
}

template <typename IO, int DK>
cudaError_t launch_simt_dk(const ScanArgs &a, cudaStream_t s) {
    constexpr size_t bytes = SimtSmem<DK>::bytes;
    auto kern = scan_simt_kernel<IO, DK>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)bytes);
    if (err != cudaSuccess) return err;
    dim3 grid(a.dv / BV, a.H, a.B);
    launch_probe_mark(s);
    kern<<<grid, NT, bytes, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

// Entry used by the C ABI: fp32 CUDA-core chunked scan for any supported shape.
cudaError_t launch_scan_simt(const ScanArgs &a, bool io_f32, cudaStream_t s) {
    if (io_f32) {
        switch (a.dk) {
            case 32: return launch_simt_dk<float, 32>(a, s);
            case 64: return launch_simt_dk<float, 64>(a, s);
            case 128: return launch_simt_dk<float, 128>(a, s);
        }
    } else {
        switch (a.dk) {
            case 32: return launch_simt_dk<__nv_bfloat16, 32>(a, s);
            case 64: return launch_simt_dk<__nv_bfloat16, 64>(a, s);
            case 128: return launch_simt_dk<__nv_bfloat16, 128>(a, s);
        }
    }
    return cudaErrorInvalidValue;
}

}  // namespace prism
