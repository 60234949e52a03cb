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
// The backward needs S_{t-1} and S_t at every token, in reverse order.  Sequential form: each CTA
// first runs the forward recurrence for its rows and writes the state at every 64-token chunk
// start to the workspace; then, chunk by chunk from the last, it recomputes the chunk's states
// from that checkpoint into a per-CTA workspace buffer (and S_{t-1} k_t into shared memory) and
// walks the chunk's tokens backwards, carrying G from chunk to chunk.  All arithmetic is fp32 from
// the exact input values.  Chunk-parallel form (bf16 I/O, dk == dv in {64, 128}): the forward's
// tensor-core scan writes the chunk-entry states, the same scan over the reversed tokens (see
// bwd_reverse_kernel) writes the gradient at every chunk end, and the CTAs, each on its own range
// of chunks, run only the recompute and reverse passes, reloading G at every chunk end.

#include <algorithm>

#include "tc.cuh"

namespace prism {

// the forward's two-kernel routes (scan_gdn.cu)
cudaError_t launch_gdn_prep(const ScanArgs &a, void *ws, cudaStream_t s);
cudaError_t launch_gdn_state(const ScanArgs &a, const void *ws, cudaStream_t s, float *ckpt);
cudaError_t launch_lrank_prep(const ScanArgs &a, void *ws, cudaStream_t s);
cudaError_t launch_lrank_state(const ScanArgs &a, const void *ws, cudaStream_t s, float *ckpt);
size_t gdn_workspace_bytes(int B, int H, int T, int dk);
size_t lrank_workspace_bytes(int B, int H, int T, int dk);

namespace {

constexpr int BW_NW = 16;              // value rows (warps) per CTA
constexpr int BW_THREADS = 32 * BW_NW;
constexpr int BW_C = 64;               // tokens between checkpoints
constexpr int BW_TB = 8;               // tokens per staged block (and per flush of the row sums)
constexpr int BW_SPC = BW_C / BW_TB;   // staged blocks per checkpoint interval

struct BwdArgs {
    int B, H, T, dk, dv, L, nch;
    const void *q, *k, *v, *u, *w, *dO;
    const float *alpha, *beta, *S0, *dS_final;
    float *dq, *dk_out, *dv_out, *dalpha, *dbeta, *du, *dw, *dS0;
    float *ckpt;     // [B, H, nch, dv, dk] state at each chunk start
    float *scratch;  // per CTA: [BW_C + 1][BW_NW][dk] states of the current chunk
    // chunk-parallel mode (ns > 0): the chunk-entry states are given in ckpt, and gexit holds the
    // gradient scan's state at each of its NR chunk starts (the gradient of the state at the end
    // of chunk c, plus that chunk's last output term, sits at NR - 1 - c); blockIdx.z = b ns + split,
    // each split walking its own contiguous range of chunks
    const float *gexit;
    int NR, ns;
};

// One staged block of BW_TB tokens (io type unless noted): k, q [TB][DK]; w [TB][L][DK];
// u [TB][L][NW] (or v [TB][NW]) and dO [TB][NW] for this CTA's NW rows; alpha, beta [TB] fp32.
template <typename IO, int DK>
struct BwdStage {
    static constexpr uint32_t K = 0;
    static constexpr uint32_t Q = K + BW_TB * DK * sizeof(IO);
    static constexpr uint32_t W = Q + BW_TB * DK * sizeof(IO);
    // u (or v: one "rank") slot, then dO, then alpha / beta; L = 0 on the Gated-DeltaNet write
    __host__ __device__ static uint32_t U(int L) { return W + BW_TB * L * DK * sizeof(IO); }
    __host__ __device__ static uint32_t DO(int L) { return U(L) + BW_TB * (L > 0 ? L : 1) * BW_NW * sizeof(IO); }
    __host__ __device__ static uint32_t AB(int L) { return DO(L) + BW_TB * BW_NW * sizeof(IO); }
    __host__ __device__ static uint32_t bytes(int L) { return (AB(L) + 2 * BW_TB * 4 + 15) & ~15u; }
};

template <typename IO, int DK>
struct BwdSmem {
    // two staged blocks; cross-row sums of a block: dq, dk, dw (L ranks), dalpha, dbeta; S_{t-1} k_t
    static size_t bytes(int L) {
        return 2 * (size_t)BwdStage<IO, DK>::bytes(L) +
               sizeof(float) * ((size_t)(2 + L) * BW_TB * DK + 2 * BW_TB + (size_t)BW_NW * BW_C);
    }
};

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(tc::smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <typename IO, int DK>
__global__ void __launch_bounds__(BW_THREADS) scan_bwd_kernel(BwdArgs p) {
    constexpr int E = DK / 32;  // columns per lane
    using SG = BwdStage<IO, DK>;
    extern __shared__ __align__(16) uint8_t smem[];
    const int L = p.L;
    const bool gdn = p.u == nullptr;
    const int Lw = gdn ? 0 : L;                       // staged write ranks
    const uint32_t SB = SG::bytes(Lw);
    float *acc_dq = reinterpret_cast<float *>(smem + 2 * SB);   // [TB][DK]
    float *acc_dk = acc_dq + BW_TB * DK;                        // [TB][DK]
    float *acc_dw = acc_dk + BW_TB * DK;                        // [TB][L][DK]
    float *acc_da = acc_dw + (size_t)BW_TB * Lw * DK;           // [TB]
    float *acc_db = acc_da + BW_TB;                             // [TB]
    float *pk_all = acc_db + BW_TB;                             // [NW][C]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r0 = blockIdx.x * BW_NW, r = r0 + warp;  // this warp's value row
    const int h = blockIdx.y, b = p.ns ? (int)blockIdx.z / p.ns : (int)blockIdx.z;
    const int split = p.ns ? (int)blockIdx.z % p.ns : 0;
    const int H = p.H, T = p.T, dv = p.dv, nch = p.nch;
    const size_t head = (size_t)b * H + h;
    const IO *q = (const IO *)p.q, *k = (const IO *)p.k, *v = (const IO *)p.v;
    const IO *u = (const IO *)p.u, *w = (const IO *)p.w, *dO = (const IO *)p.dO;
    float *pk = pk_all + warp * BW_C;
    const size_t cta = ((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
    float *scr = p.scratch + cta * (size_t)(BW_C + 1) * BW_NW * DK + warp * DK;  // + i * NW * DK
    auto tok = [&](int t) { return ((size_t)b * T + t) * H + h; };  // index of (b, t, h)
    auto ckpt_row = [&](int c) { return p.ckpt + (((head * nch + c) * dv) + r) * DK; };

    // ---- staging of token blocks (cp.async, all threads)
    const int nsb = (T + BW_TB - 1) / BW_TB;
    auto stage = [&](int buf, int sb) {
        uint8_t *st = smem + buf * SB;
        const int t0 = sb * BW_TB, m = min(BW_TB, T - t0);
        constexpr int RC = DK * sizeof(IO) / 16;          // 16-byte pieces of a k / q / w row
        constexpr int NC = BW_NW * sizeof(IO) / 16;       // pieces of a 16-row slice
        const int nk = m * RC, nw = m * Lw * RC, nu = m * Lw * NC, nd = m * NC;
        const int nv = gdn ? m * NC : 0;
        const int total = 2 * nk + nw + nu + nd + nv + 2 * m;
        for (int e = tid; e < total; e += BW_THREADS) {
            int x = e;
            if (x < 2 * nk) {  // k, q rows
                const int which = x / nk, y = x % nk, i = y / RC, pc = y % RC;
                const IO *src = (which ? q : k) + tok(t0 + i) * DK;
                cp_async16(st + (which ? SG::Q : SG::K) + (i * DK) * sizeof(IO) + pc * 16,
                           reinterpret_cast<const uint8_t *>(src) + pc * 16);
                continue;
            }
            x -= 2 * nk;
            if (x < nw) {  // w rows
                const int i = x / (Lw * RC), l = (x / RC) % Lw, pc = x % RC;
                cp_async16(st + SG::W + ((i * Lw + l) * DK) * sizeof(IO) + pc * 16,
                           reinterpret_cast<const uint8_t *>(w + (tok(t0 + i) * L + l) * DK) + pc * 16);
                continue;
            }
            x -= nw;
            if (x < nu) {  // u slices of this CTA's rows
                const int i = x / (Lw * NC), l = (x / NC) % Lw, pc = x % NC;
                cp_async16(st + SG::U(Lw) + ((i * Lw + l) * BW_NW) * sizeof(IO) + pc * 16,
                           reinterpret_cast<const uint8_t *>(u + (tok(t0 + i) * L + l) * dv + r0) + pc * 16);
                continue;
            }
            x -= nu;
            if (x < nd + nv) {  // dO slices, then v slices (into the u slot on the GDN write)
                const bool isv = x >= nd;
                const int y = isv ? x - nd : x, i = y / NC, pc = y % NC;
                const IO *src = (isv ? v : dO) + tok(t0 + i) * dv + r0;
                cp_async16(st + (isv ? SG::U(Lw) : SG::DO(Lw)) + (i * BW_NW) * sizeof(IO) + pc * 16,
                           reinterpret_cast<const uint8_t *>(src) + pc * 16);
                continue;
            }
            x -= nd + nv;
            {  // alpha, beta
                const int which = x / m, i = x % m;
                cp_async4(st + SG::AB(Lw) + (which * BW_TB + i) * 4, (which ? p.beta : p.alpha) + tok(t0 + i));
            }
        }
    };
    // staged values of token i of the block in buffer `buf`
    auto sk = [&](int buf, int i, int c) { return ld_io<IO>((const IO *)(smem + buf * SB + SG::K), i * DK + c); };
    auto sq = [&](int buf, int i, int c) { return ld_io<IO>((const IO *)(smem + buf * SB + SG::Q), i * DK + c); };
    auto sw = [&](int buf, int i, int l, int c) {
        return ld_io<IO>((const IO *)(smem + buf * SB + SG::W), (i * Lw + l) * DK + c);
    };
    auto su = [&](int buf, int i, int l) {  // u_{t,l} of this warp's row (v_t on the GDN write)
        return ld_io<IO>((const IO *)(smem + buf * SB + SG::U(Lw)), (i * (gdn ? 1 : Lw) + l) * BW_NW + warp);
    };
    auto sdo = [&](int buf, int i) { return ld_io<IO>((const IO *)(smem + buf * SB + SG::DO(Lw)), i * BW_NW + warp); };
    auto sa = [&](int buf, int i) { return reinterpret_cast<const float *>(smem + buf * SB + SG::AB(Lw))[i]; };
    auto sbeta = [&](int buf, int i) { return reinterpret_cast<const float *>(smem + buf * SB + SG::AB(Lw))[BW_TB + i]; };

    auto dot = [&](const float (&a)[E], const float (&c)[E]) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < E; ++i) s = fmaf(a[i], c[i], s);
        return warp_sum(s);
    };
    // one forward step of this warp's row at staged token i; returns S_{t-1} k_t of the row
    auto step = [&](float (&s)[E], int buf, int i) -> float {
        float kk[E];
#pragma unroll
        for (int e = 0; e < E; ++e) kk[e] = sk(buf, i, lane + 32 * e);
        const float sk_ = dot(s, kk);
        const float a = sa(buf, i), be = sbeta(buf, i);
#pragma unroll
        for (int e = 0; e < E; ++e) s[e] = a * fmaf(-be * sk_, kk[e], s[e]);
        if (gdn) {
            const float bv = be * su(buf, i, 0);
#pragma unroll
            for (int e = 0; e < E; ++e) s[e] = fmaf(bv, kk[e], s[e]);
        } else {
            for (int l = 0; l < L; ++l) {
                const float ur = su(buf, i, l);
#pragma unroll
                for (int e = 0; e < E; ++e) s[e] = fmaf(ur, sw(buf, i, l, lane + 32 * e), s[e]);
            }
        }
        return sk_;
    };
    auto store_state = [&](float *dst, const float (&s)[E]) {
#pragma unroll
        for (int i = 0; i < E; ++i) dst[lane + 32 * i] = s[i];
    };
    auto load_state = [&](const float *src, float (&s)[E]) {
#pragma unroll
        for (int i = 0; i < E; ++i) s[i] = src[lane + 32 * i];
    };

    // ---- the schedule: the forward sweep over every block, then for each checkpoint interval from
    // the last: its blocks forwards (recomputing the states), then backwards
    enum { kFwd, kRecomp, kRev };
    const int last_sb = (nch - 1) * BW_SPC, m_last = nsb - last_sb;  // blocks of the last interval
    // chunk-parallel mode: no forward sweep, and this CTA's chunks [c_lo, c_hi) only
    const int c_lo = p.ns ? (int)((long long)nch * split / p.ns) : 0;
    const int c_hi = p.ns ? (int)((long long)nch * (split + 1) / p.ns) : nch;
    const int fwd = p.ns ? 0 : nsb;  // forward-sweep steps
    auto schedule = [&](int j, int &sb, int &mode) {
        if (j < fwd) { sb = j; mode = kFwd; return; }
        int j2 = j - fwd, c, kk, m;
        if (c_hi < nch) j2 += 2 * m_last + 2 * BW_SPC * (nch - 1 - c_hi);  // skip the later chunks
        if (j2 < 2 * m_last) {
            c = nch - 1; kk = j2; m = m_last;
        } else {
            const int jj = j2 - 2 * m_last;
            c = nch - 2 - jj / (2 * BW_SPC); kk = jj % (2 * BW_SPC); m = BW_SPC;
        }
        mode = kk < m ? kRecomp : kRev;
        sb = c * BW_SPC + (kk < m ? kk : 2 * m - 1 - kk);
    };
    const int steps = p.ns ? (c_hi <= c_lo ? 0
                                          : (c_hi == nch ? 2 * m_last + 2 * BW_SPC * (nch - 1 - c_lo)
                                                         : 2 * BW_SPC * (c_hi - c_lo)))
                           : 3 * nsb;

    float s[E], g[E];
    if (p.S0) load_state(p.S0 + (head * dv + r) * DK, s);
    else {
#pragma unroll
        for (int i = 0; i < E; ++i) s[i] = 0.f;
    }
    if (p.dS_final) load_state(p.dS_final + (head * dv + r) * DK, g);
    else {
#pragma unroll
        for (int i = 0; i < E; ++i) g[i] = 0.f;
    }
    const int acc_n = (2 + Lw) * BW_TB * DK + 2 * BW_TB;
    for (int e = tid; e < acc_n; e += BW_THREADS) acc_dq[e] = 0.f;

    if (steps > 0) {
        int sb0, md0;
        schedule(0, sb0, md0);
        stage(0, sb0);
    }
    cp_async_commit();
    for (int j = 0; j < steps; ++j) {
        const int buf = j & 1;
        if (j + 1 < steps) {
            int sbn, mdn;
            schedule(j + 1, sbn, mdn);
            stage(buf ^ 1, sbn);
        }
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        int sb, mode;
        schedule(j, sb, mode);
        const int t0 = sb * BW_TB, m = min(BW_TB, T - t0);
        const int c = sb / BW_SPC, ci0 = (sb % BW_SPC) * BW_TB;  // interval, first index in it
        if (mode == kFwd) {
            if (ci0 == 0) store_state(ckpt_row(c), s);
            for (int i = 0; i < m; ++i) step(s, buf, i);
        } else if (mode == kRecomp) {
            if (ci0 == 0) {
                load_state(ckpt_row(c), s);
                store_state(scr, s);
                if (p.ns) {
                    // the gradient at the chunk's end from everything after it: the gradient scan's
                    // state there less the chunk's last output term, which the reverse pass adds
                    load_state(p.gexit + ((head * p.NR + (p.NR - 1 - c)) * dv + r) * DK, g);
                    const int tl = (c + 1) * BW_C - 1;
                    if (tl < T) {
                        const float dd = ld_io<IO>(dO, tok(tl) * dv + r);
#pragma unroll
                        for (int e = 0; e < E; ++e) g[e] -= dd * ld_io<IO>(q, tok(tl) * DK + lane + 32 * e);
                    }
                }
            }
            for (int i = 0; i < m; ++i) {
                const float pki = step(s, buf, i);
                if (lane == 0) pk[ci0 + i] = pki;
                store_state(scr + (size_t)(ci0 + i + 1) * BW_NW * DK, s);
            }
        } else {
            __syncwarp();
            // the block's states S_{t0-1} .. S_{t0+m-1} of this row, all loads issued at once
            float st[BW_TB + 1][E];
#pragma unroll
            for (int i = 0; i <= BW_TB; ++i)
                if (i <= m) load_state(scr + (size_t)(ci0 + i) * BW_NW * DK, st[i]);
#pragma unroll
            for (int i = BW_TB - 1; i >= 0; --i) {
                if (i >= m) continue;
                const int t = t0 + i;
                float kk[E], qq[E];
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    kk[e] = sk(buf, i, lane + 32 * e);
                    qq[e] = sq(buf, i, lane + 32 * e);
                }
                const float dd = sdo(buf, i);
                const float a = sa(buf, i), be = sbeta(buf, i);
                const float Pk = pk[ci0 + i];
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    g[e] = fmaf(dd, qq[e], g[e]);
                    atomicAdd(&acc_dq[i * DK + lane + 32 * e], dd * st[i + 1][e]);
                }
                const float Gk = dot(g, kk), gs = dot(g, st[i]);
                float da = gs - be * Pk * Gk, db = -a * Pk * Gk;
                const float ab = a * be;
                float dk_[E];
#pragma unroll
                for (int e = 0; e < E; ++e) dk_[e] = -ab * fmaf(g[e], Pk, st[i][e] * Gk);
                if (gdn) {
                    const float vr = su(buf, i, 0);
                    db = fmaf(vr, Gk, db);
#pragma unroll
                    for (int e = 0; e < E; ++e) dk_[e] = fmaf(be * vr, g[e], dk_[e]);
                    if (lane == 0) p.dv_out[tok(t) * dv + r] = be * Gk;
                } else {
                    for (int l = 0; l < L; ++l) {
                        float ww[E];
#pragma unroll
                        for (int e = 0; e < E; ++e) ww[e] = sw(buf, i, l, lane + 32 * e);
                        const float ur = su(buf, i, l);
                        const float dul = dot(g, ww);
                        if (lane == 0) p.du[(tok(t) * L + l) * dv + r] = dul;
#pragma unroll
                        for (int e = 0; e < E; ++e)
                            atomicAdd(&acc_dw[((size_t)i * Lw + l) * DK + lane + 32 * e], ur * g[e]);
                    }
                }
#pragma unroll
                for (int e = 0; e < E; ++e) atomicAdd(&acc_dk[i * DK + lane + 32 * e], dk_[e]);
                if (lane == 0) {
                    atomicAdd(&acc_da[i], da);
                    atomicAdd(&acc_db[i], db);
                }
#pragma unroll
                for (int e = 0; e < E; ++e) g[e] = a * fmaf(-be * Gk, kk[e], g[e]);
            }
            // the block's row sums from this CTA into the global gradients, then clear them
            __syncthreads();
            for (int e = tid; e < m * DK; e += BW_THREADS) {
                const int sl = e / DK, jc = e % DK;
                const size_t o = tok(t0 + sl) * DK + jc;
                atomicAdd(&p.dq[o], acc_dq[e]);
                atomicAdd(&p.dk_out[o], acc_dk[e]);
                acc_dq[e] = 0.f;
                acc_dk[e] = 0.f;
            }
            for (int e = tid; e < m * Lw * DK; e += BW_THREADS) {
                const int sl = e / (Lw * DK), l = (e / DK) % Lw, jc = e % DK;
                atomicAdd(&p.dw[(tok(t0 + sl) * L + l) * DK + jc], acc_dw[e]);
                acc_dw[e] = 0.f;
            }
            if (tid < m) {
                atomicAdd(&p.dalpha[tok(t0 + tid)], acc_da[tid]);
                atomicAdd(&p.dbeta[tok(t0 + tid)], acc_db[tid]);
                acc_da[tid] = 0.f;
                acc_db[tid] = 0.f;
            }
        }
        __syncthreads();  // the block's buffer is free for the block two steps ahead
    }
    cp_async_wait<0>();
    if (p.dS0 && !p.ns) store_state(p.dS0 + (head * dv + r) * DK, g);
}

// The gradient scan's inputs (chunk-parallel backward).  With G_t the gradient of the state after
// token t (0-indexed tokens; G_{T-1} = dS_final + dO_{T-1} q_{T-1}^T, G_{t-1} = G_t A_t +
// dO_{t-1} q_{t-1}^T, A_t = alpha_t (I - beta_t k_t k_t^T), dS0 = G_{-1} = G_0 A_0), the gradient
// runs as the scan's own recurrence over the tokens in reverse: position P + i carries token
// T - 1 - i's transition and the rank-1 write u = dO, w = q of the token before it (none for
// i = T - 1).  P = 64 - T % 64 positions in front (identity transitions; the last of them writes
// dO_{T-1} q_{T-1}^T onto the entry state dS_final) align the scan's 64-token chunks with the
// forward's chunk ends.  One thread a 16-byte piece of a row; bf16 rows are copied bit for bit.
template <typename IO>
__global__ void __launch_bounds__(128) bwd_reverse_kernel(int B, int T, int H, int dk, int dv, int P,
                                                          const IO *q, const IO *k, const float *alpha,
                                                          const float *beta, const IO *dO, IO *kr,
                                                          IO *ur, IO *wr, float *ar, float *br) {
    const int Tp = T + P;
    const long long idx = blockIdx.x;  // (b, position, h)
    const int h = (int)(idx % H), pos = (int)((idx / H) % Tp), b = (int)(idx / ((long long)H * Tp));
    int tk = -1, tw = -1;  // source tokens of the transition and of the write
    if (pos == P - 1) tw = T - 1;
    else if (pos >= P) {
        tk = T - 1 - (pos - P);
        tw = tk - 1;
    }
    auto src = [&](int t) { return ((size_t)b * T + t) * H + h; };
    const size_t dst = idx;  // ((b Tp + pos) H + h)
    constexpr int PER = 16 / (int)sizeof(IO);
    const uint4 zero = make_uint4(0, 0, 0, 0);
    for (int c = threadIdx.x; c < dk / PER; c += blockDim.x) {
        reinterpret_cast<uint4 *>(kr + dst * dk)[c] = tk >= 0 ? reinterpret_cast<const uint4 *>(k + src(tk) * dk)[c] : zero;
        reinterpret_cast<uint4 *>(wr + dst * dk)[c] = tw >= 0 ? reinterpret_cast<const uint4 *>(q + src(tw) * dk)[c] : zero;
    }
    for (int c = threadIdx.x; c < dv / PER; c += blockDim.x)
        reinterpret_cast<uint4 *>(ur + dst * dv)[c] = tw >= 0 ? reinterpret_cast<const uint4 *>(dO + src(tw) * dv)[c] : zero;
    if (threadIdx.x == 0) {
        ar[dst] = tk >= 0 ? alpha[src(tk)] : 1.f;
        br[dst] = tk >= 0 ? beta[src(tk)] : 0.f;
    }
}

template <typename IO, int DK>
cudaError_t launch_bwd_t(const BwdArgs &a, cudaStream_t s) {
    const size_t bytes = BwdSmem<IO, DK>::bytes(a.u == nullptr ? 0 : a.L);
    auto kern = scan_bwd_kernel<IO, DK>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (err != cudaSuccess) return err;
    dim3 grid(a.dv / BW_NW, a.H, a.B * (a.ns ? a.ns : 1));
    launch_probe_mark(s);
    kern<<<grid, BW_THREADS, bytes, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

// The chunk-parallel backward (bf16 I/O on the tensor-core shapes): the forward scan writes every
// chunk's entry state, the gradient scan (the forward's own kernels on the reversed tokens, above)
// writes the gradient at every chunk end, and then every chunk's token-level reverse pass runs on
// its own, split into ns ranges of chunks per sequence so that the grid fills the GPU several times.
namespace {

bool chunked_bwd(int dk, int dv, bool io_f32) { return !io_f32 && dk == dv && (dk == 64 || dk == 128); }

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
        return 148;
    return n;
}

int bwd_splits(int B, int H, int dv, int nch) {
    const long long base = (long long)B * H * (dv / BW_NW);  // CTAs of one split
    const long long want = (8LL * sm_count() + base - 1) / base;
    return (int)std::max(1LL, std::min<long long>({want, (long long)nch, 65535LL / std::max(B, 1)}));
}

struct BwdLayout {  // byte offsets into the workspace
    size_t ckpt, gexit, scratch, kr, ur, wr, ar, br, rec, total;
    int nch, P, Tp, NR, ns;
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

BwdLayout bwd_layout(int B, int H, int T, int dk, int dv, bool io_f32) {
    BwdLayout l{};
    l.nch = (T + BW_C - 1) / BW_C;
    const size_t heads = (size_t)B * H, st = (size_t)dv * dk * sizeof(float);
    const bool chunked = chunked_bwd(dk, dv, io_f32) && T > 0;
    l.ns = chunked ? bwd_splits(B, H, dv, l.nch) : 0;
    l.P = BW_C - T % BW_C;  // 1 .. 64 identity positions in front of the reversed tokens
    l.Tp = T + l.P;
    l.NR = l.Tp / BW_C;
    size_t o = kStatusBytes;
    l.ckpt = o;
    o = align256(o + heads * l.nch * st);
    const size_t ctas = heads * (dv / BW_NW) * (size_t)(l.ns ? l.ns : 1);
    l.scratch = o;
    o = align256(o + ctas * (BW_C + 1) * BW_NW * dk * sizeof(float));
    if (chunked) {
        const size_t ntok = heads * l.Tp, io = 2;
        l.gexit = o;
        o = align256(o + heads * l.NR * st);
        l.kr = o;
        o = align256(o + ntok * dk * io);
        l.ur = o;
        o = align256(o + ntok * dv * io);
        l.wr = o;
        o = align256(o + ntok * dk * io);
        l.ar = o;
        o = align256(o + ntok * sizeof(float));
        l.br = o;
        o = align256(o + ntok * sizeof(float));
        // the forward's records (either write form), then the gradient scan's, in one region
        l.rec = o;
        const size_t rec = std::max({gdn_workspace_bytes(B, H, T, dk), lrank_workspace_bytes(B, H, T, dk),
                                     lrank_workspace_bytes(B, H, l.Tp, dk)});
        o = align256(o + rec);
    }
    l.total = o;
    return l;
}

}  // namespace

// Workspace of the backward after the status block: the chunk-start states of every row, one
// chunk of states per CTA, and for the chunk-parallel form the gradient scan's chunk states, its
// inputs and the scans' records.
size_t bwd_workspace_bytes(int B, int H, int T, int dk, int dv, bool io_f32) {
    return bwd_layout(B, H, T, dk, dv, io_f32).total;
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
    const BwdLayout lay = bwd_layout(f.B, f.H, f.T, f.dk, f.dv, io_f32);
    uint8_t *wb = (uint8_t *)ws;
    a.ckpt = (float *)(wb + lay.ckpt);
    a.scratch = (float *)(wb + lay.scratch);
    a.gexit = nullptr;
    a.NR = 0;
    a.ns = 0;
    if (lay.ns) {
        // 1. the forward over the same tokens, keeping every chunk's entry state (no outputs)
        ScanArgs fa = f;
        fa.o = nullptr;
        fa.S_final = nullptr;
        fa.flags = kNoOutput;
        void *rec = wb + lay.rec;
        const bool gdn = f.u == nullptr;
        if ((err = gdn ? launch_gdn_prep(fa, rec, s) : launch_lrank_prep(fa, rec, s)) != cudaSuccess) return err;
        if ((err = gdn ? launch_gdn_state(fa, rec, s, a.ckpt) : launch_lrank_state(fa, rec, s, a.ckpt)) != cudaSuccess)
            return err;
        // 2. the gradient scan's inputs, then the scan itself (rank-1 write), which leaves the
        //    gradient at every chunk end in gexit and dS0 in its exit state
        const __nv_bfloat16 *qb = (const __nv_bfloat16 *)f.q, *kb = (const __nv_bfloat16 *)f.k;
        __nv_bfloat16 *kr = (__nv_bfloat16 *)(wb + lay.kr), *ur = (__nv_bfloat16 *)(wb + lay.ur),
                      *wr = (__nv_bfloat16 *)(wb + lay.wr);
        float *ar = (float *)(wb + lay.ar), *br = (float *)(wb + lay.br);
        launch_probe_mark(s);
        bwd_reverse_kernel<__nv_bfloat16><<<(unsigned)((size_t)f.B * lay.Tp * f.H), 128, 0, s>>>(
            f.B, f.T, f.H, f.dk, f.dv, lay.P, qb, kb, f.alpha, f.beta, (const __nv_bfloat16 *)dO, kr, ur, wr,
            ar, br);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        ScanArgs ra = f;
        ra.T = lay.Tp;
        ra.L = 1;
        ra.q = kr;
        ra.k = kr;
        ra.v = kr;  // (not read by the rank-L write; dv == dk)
        ra.alpha = ar;
        ra.beta = br;
        ra.u = ur;
        ra.w = wr;
        ra.S0 = dS_final;
        ra.o = nullptr;
        ra.S_final = dS0;
        ra.flags = kNoOutput;
        float *gexit = (float *)(wb + lay.gexit);
        if ((err = launch_lrank_prep(ra, rec, s)) != cudaSuccess) return err;
        if ((err = launch_lrank_state(ra, rec, s, gexit)) != cudaSuccess) return err;
        // 3. every chunk's own gradients from (its entry state, the gradient at its end)
        a.gexit = gexit;
        a.NR = lay.NR;
        a.ns = lay.ns;
        a.dS0 = nullptr;  // written by the gradient scan
    }
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
