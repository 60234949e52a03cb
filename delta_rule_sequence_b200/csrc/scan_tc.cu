// scan_tc.cu -- chunked scan forward on the tcgen05 tensor cores (bf16 operands, fp32 TMEM
// accumulators, fp32 state).
//
// One CTA owns one (batch, head, slice of BV value rows) sequence and walks its chunks of C = 64
// tokens in order.  Rows of the state evolve independently, so value slices need no
// communication.  The fp32 state lives in registers as S^T (thread <-> key index d, BV values).
//
// Per chunk (notation of "Sequential Parallel Duality in Prefix Scannable Models", method
// overview: chunk, encode, scan; the chunk form is exact because the per-token affine elements
// E_t = alpha_t (I - beta_t k_t k_t^T), f_t = sum_l u w^T compose associatively), with entry state
// S and g_t = sum_{r<=t} log alpha_r, Gamma_{t,i} = e^{g_t - g_i}, D_i = e^{g_n - g_i}:
//   G      = [K; Q] K^T                                  tensor core, M = 128
//   A      = strict(diag(beta) Gamma o K K^T)  Mqk = incl(Gamma o Q K^T)      CUDA cores
//   T      = (I + A)^{-1}                                  blocked fp32 substitution
//   Wk     = T diag(beta e^g) K                           tensor core (the WY / UT transform)
//   Gated-DeltaNet write (u = beta v, w = k):  U = T diag(beta) V,  Y = U - Wk S^T
//   rank-L write: P_l = strict(diag(beta) Gamma o K W_l^T), Mqw_l = incl(Gamma o Q W_l^T),
//     X_u = T sum_l P_l U_l,  Y = -(X_u + Wk S^T),  O_w = sum_l Mqw_l U_l,
//     F_w = sum_l W_l^T D U_l
//   O      = diag(e^g) Q S^T + Mqk Y (+ O_w)
//   S'^T   = e^{g_n} S^T + K^T D Y (+ F_w)
// which is the token recurrence S_t = alpha_t S_{t-1}(I - beta_t k_t k_t^T) + sum_l u_{t,l}
// w_{t,l}^T, o_t = S_t q_t (PRISM, gist.science explainer, technical summary 2.1 and 2.2)
// unrolled over the chunk.  Every matrix product is a tcgen05.mma issued by one thread from
// shared-memory operands in the canonical 128B/64B-swizzled layouts; accumulators are read back
// with tcgen05.ld.  Waits on MMA completion are bounded and record PRISM_ERR_TIMEOUT.

#include "chunk_common.cuh"

namespace prism {
namespace {

constexpr int NT = 128;       // 4 warps: TMEM lanes 0-127
constexpr uint32_t TMEM_COLS = 512;

// Operands that are rounded intermediate results (Mqk, T, Y, S and, for the rank-L write, P, Mqw,
// D U, sum P U) are kept as an unevaluated bf16 pair x = hi + lo (lo = bf16(x - hi)); a product
// a b is then formed as a_hi b_hi + a_hi b_lo + a_lo b_hi by extra MMAs into the same TMEM
// accumulator, which carries about 16 significant bits instead of 8.  The inputs q, k, v, u, w
// are exact bf16 already and are used as they are.
template <int DK, int BV, bool GDN>
struct TcLayout {
    static constexpr uint32_t KB = 1024;
    static constexpr uint32_t KQW_BLK = 3 * C * 128;           // [K; Q; Wk] rows of one 64-col block
    static constexpr uint32_t KQW = 0;
    static constexpr uint32_t ROWB = (BV == 32) ? 64 : 128;    // bytes per row of an x BV tile
    static constexpr uint32_t VT = C * ROWB;                   // C x BV bf16 tile
    static constexpr uint32_t SQ = C * 128;                    // C x C bf16 tile
    static constexpr uint32_t W_BLK = C * 128;
    static constexpr uint32_t V = KQW + KQW_BLK * (DK / 64);   // V slice (GDN) or U_l slice
    static constexpr uint32_t DU = V + VT;                     // D U_l hi, lo (rank-L)
    static constexpr uint32_t DUL = DU + (GDN ? 0 : VT);
    static constexpr uint32_t W = DUL + (GDN ? 0 : VT);        // W_l, C x DK K-major (rank-L)
    static constexpr uint32_t T1 = W + (GDN ? 0 : W_BLK * (DK / 64));
    static constexpr uint32_t T1L = T1 + SQ;
    static constexpr uint32_t T2 = T1L + SQ;
    static constexpr uint32_t T2L = T2 + SQ;
    static constexpr uint32_t MQK = T2L + SQ;
    static constexpr uint32_t MQKL = MQK + SQ;
    static constexpr uint32_t PU = MQKL + SQ;                  // sum_l P_l U_l hi, lo (rank-L)
    static constexpr uint32_t PUL = PU + (GDN ? 0 : VT);
    static constexpr uint32_t S = PUL + (GDN ? 0 : VT);        // S^T [d][v] hi, lo
    static constexpr uint32_t SL = S + DK * ROWB;
    static constexpr uint32_t Y = SL + DK * ROWB;
    static constexpr uint32_t YL = Y + VT;
    static constexpr uint32_t DY = YL + VT;
    static constexpr uint32_t DYL = DY + VT;
    // fp32 solve buffers; after the bf16 T tiles are built the rank-L P / Mqw tiles reuse them
    static constexpr uint32_t AF = DYL + VT;                   // fp32 A  [C][AS]
    static constexpr uint32_t TF = AF + C * AS * 4;            // fp32 T  [C][AS]
    static constexpr uint32_t TMP = TF + C * AS * 4;           // fp32 32 x 33 scratch
    static constexpr uint32_t P = AF;                          // P_l hi, lo; Mqw_l hi, lo
    static constexpr uint32_t PL = P + SQ;
    static constexpr uint32_t MQW = PL + SQ;
    static constexpr uint32_t MQWL = MQW + SQ;
    static_assert(MQWL + SQ <= TMP + 32 * 33 * 4, "P / Mqw tiles must fit the solve buffers");
    static constexpr uint32_t GATES = TMP + 32 * 33 * 4;       // g, beta, gamma, D: 4 x C floats
    static constexpr uint32_t END = GATES + 4 * C * 4;
    static constexpr uint32_t BYTES = ((END + KB - 1) / KB) * KB + KB;  // + alignment slack
    // TMEM columns
    static constexpr uint32_t cG = 0;            // [K;Q] K^T or [K;Q] W_l^T   (64 columns)
    static constexpr uint32_t cWk = 64;          // Wk                          (DK columns)
    static constexpr uint32_t cU = cWk + DK;     // U (GDN) or X_u (rank-L)     (BV)
    static constexpr uint32_t cPU = cU + BV;     // sum_l P_l U_l               (BV)
    static constexpr uint32_t cO = cPU + BV;     // O_w + Mqk Y                 (BV)
    static constexpr uint32_t cXs = cO + BV;     // Wk S^T                      (BV)
    static constexpr uint32_t cQS = cXs + BV;    // Q S^T                       (BV)
    static constexpr uint32_t cDS = cQS + BV;    // F_w + K^T D Y               (BV)
    static_assert(cDS + BV <= TMEM_COLS, "TMEM budget");
};

template <int DK, int BV, bool GDN>
__global__ void __launch_bounds__(NT, 1) scan_tc_kernel(ScanArgs p) {
    using LY = TcLayout<DK, BV, GDN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t mma_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int failed_sh;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int v0 = blockIdx.x * BV, h = blockIdx.y, b = blockIdx.z;
    const int H = p.H, T = p.T, dv = p.dv, L = GDN ? 1 : p.L;
    const bool wr = !(p.flags & kNoWrite);  // the write term is present
    const bool rank_l = !GDN && wr;         // the rank-L terms X_u, O_w, F_w are present
    const __nv_bfloat16 *q = (const __nv_bfloat16 *)p.q, *k = (const __nv_bfloat16 *)p.k;
    const __nv_bfloat16 *v = (const __nv_bfloat16 *)p.v, *u = (const __nv_bfloat16 *)p.u;
    const __nv_bfloat16 *w = (const __nv_bfloat16 *)p.w;
    __nv_bfloat16 *o = (__nv_bfloat16 *)p.o;
    const size_t head = (size_t)b * H + h;

    float *sA = (float *)(sm + LY::AF);
    float *sTmp = (float *)(sm + LY::TMP);
    float *sG = (float *)(sm + LY::GATES);
    float *sBeta = sG + C;
    float *sGam = sBeta + C;
    float *sD = sGam + C;
    const uint32_t sb = smem_u32(sm);

    if (warp == 0) tmem_alloc(&tmem_base_sh, TMEM_COLS);
    if (tid == 0) {
        mbar_init(&mma_bar, 1);
        mbar_fence_init();
        failed_sh = 0;
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tb = tmem_base_sh;
    uint32_t phase = 0;

    // thread 0 has issued MMAs: commit them and let every thread wait (bounded) for completion
    auto mma_done = [&]() -> bool {
        if (tid == 0) mma_commit(&mma_bar);
        __syncwarp();
        const bool ok = mbar_wait(&mma_bar, phase & 1, p.status);
        phase++;
        if (!ok) failed_sh = 1;
        fence_after_sync();
        __syncthreads();
        return failed_sh == 0;
    };
    auto dK = [](uint32_t base, int ks) { return desc_k_sw128(base, ks, 0); };          // C x C
    auto dKQW = [](uint32_t base, int ks) { return desc_k_sw128(base, ks, LY::KQW_BLK); };
    auto dKmn = [](uint32_t base, int ks) { return desc_mn_sw128(base, ks, LY::KQW_BLK); };
    auto dWmn = [](uint32_t base, int ks) { return desc_mn_sw128(base, ks, LY::W_BLK); };
    auto dVT = [](uint32_t base, int ks) { return desc_vt<BV>(base, ks); };

    // fp32 state S^T in registers: DK = 128 -> d = tid (M = 128 rows); DK = 64 -> M = 64 layout
    const bool own_d = (DK == 128) ? true : (lane < 16);
    const int d_row = (DK == 128) ? tid : (16 * warp + lane);
    float Sreg[BV];
#pragma unroll
    for (int j = 0; j < BV; ++j) Sreg[j] = 0.f;
    if (own_d && (p.flags & kS0Identity)) {
#pragma unroll
        for (int j = 0; j < BV; ++j) Sreg[j] = (v0 + j == d_row) ? 1.f : 0.f;
    } else if (own_d && p.S0) {
#pragma unroll
        for (int j = 0; j < BV; ++j) Sreg[j] = p.S0[(head * dv + v0 + j) * DK + d_row];
    }
    if (own_d) store_row_split<BV>(sm + LY::S, sm + LY::SL, d_row, Sreg);

    // M = 64 accumulators: thread (warp, lane < 16) holds chunk row 16 warp + lane
    const bool own_t = lane < 16;
    const int t_row = 16 * warp + lane;

    for (int c0 = 0; c0 < T; c0 += C) {
        const int n = min(C, T - c0);
        // ---- inputs: K, Q (rows >= n are zero: identity tokens), V slice, gates
        for (int e = tid; e < C * (DK / 8); e += NT) {
            const int t = e / (DK / 8), ch = e % (DK / 8);
            uint4 kv = make_uint4(0, 0, 0, 0), qv = kv;
            if (t < n) {
                const size_t g = (((size_t)b * T + c0 + t) * H + h) * DK + ch * 8;
                kv = *reinterpret_cast<const uint4 *>(k + g);
                qv = *reinterpret_cast<const uint4 *>(q + g);
            }
            st16(sm + LY::KQW, sw128_off(t, ch * 8, LY::KQW_BLK), kv);
            st16(sm + LY::KQW, sw128_off(C + t, ch * 8, LY::KQW_BLK), qv);
        }
        if constexpr (GDN) {
            for (int e = tid; e < C * (BV / 8); e += NT) {
                const int t = e / (BV / 8), ch = e % (BV / 8);
                uint4 vv = make_uint4(0, 0, 0, 0);
                if (t < n) {
                    const size_t g = (((size_t)b * T + c0 + t) * H + h) * dv + v0 + ch * 8;
                    vv = *reinterpret_cast<const uint4 *>(v + g);
                }
                st16(sm + LY::V, vt_off<BV>(t, ch * 8), vv);
            }
        }
        if (tid < C) {
            const size_t bth = ((size_t)b * T + c0 + tid) * H + h;
            sG[tid] = tid < n ? logf(p.alpha[bth]) : 0.f;
            sBeta[tid] = tid < n ? p.beta[bth] : 0.f;
        }
        __syncthreads();
        if (warp == 0) {
            const float x0 = warp_inclusive_scan(sG[lane], lane);
            const float x1 = warp_inclusive_scan(sG[32 + lane], lane) + __shfl_sync(0xffffffffu, x0, 31);
            sG[lane] = x0;
            sG[32 + lane] = x1;
        }
        __syncthreads();
        const float g_last = sG[C - 1];
        if (tid < C) {
            sGam[tid] = expf(sG[tid]);
            sD[tid] = tid < n ? expf(g_last - sG[tid]) : 0.f;
        }
        sync_for_mma();

        // ---- G = [K; Q] K^T ; A and Mqk
        if (tid == 0)
            mma_split(tb + LY::cG, idesc_bf16(128, C, 0, 0), DK / 16, dKQW, dKQW, sb + LY::KQW, 0,
                      sb + LY::KQW, 0, false);
        if (!mma_done()) break;
        {
            const int t = (warp & 1) * 32 + lane;  // row of K K^T (warps 0-1) or Q K^T (2-3)
            const float gt = sG[t], bt = sBeta[t];
#pragma unroll
            for (int c = 0; c < C; c += 32) {
                float gr[32];
                tmem_ld32(taddr(tb, 32 * warp, LY::cG + c), gr);
                tmem_wait_ld();
                if (warp < 2) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int i = c + j;
                        sA[t * AS + i] = (i < t) ? bt * expf(gt - sG[i]) * gr[j] : 0.f;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int i = c + j;
                        gr[j] = (i <= t) ? expf(gt - sG[i]) * gr[j] : 0.f;
                    }
                    store32_split(sm + LY::MQK, sm + LY::MQKL, t, c, gr);
                }
            }
        }
        __syncthreads();

        // ---- T = (I + A)^{-1}; bf16 pairs of T diag(beta gamma) and T diag(beta) (GDN) or T
        solve_unit_lower<NT>(sA, sA, sTmp, tid);  // in place: sA now holds T
        for (int e = tid; e < C * (C / 8); e += NT) {
            const int t = e / (C / 8), c8 = e % (C / 8);
            float a1[8], a2[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = c8 * 8 + j;
                const float tv = (i <= t) ? sA[t * AS + i] : 0.f;
                a1[j] = tv * sBeta[i] * sGam[i];
                a2[j] = GDN ? tv * sBeta[i] : tv;
            }
            uint4 h1, l1, h2, l2;
            split8(a1, h1, l1);
            split8(a2, h2, l2);
            const uint32_t off = sw128_off(t, c8 * 8, 0);
            st16(sm + LY::T1, off, h1);
            st16(sm + LY::T1L, off, l1);
            st16(sm + LY::T2, off, h2);
            st16(sm + LY::T2L, off, l2);
        }
        sync_for_mma();

        // ---- Wk = T diag(beta gamma) K ; GDN: U = T diag(beta) V
        if (tid == 0) {
            mma_split(tb + LY::cWk, idesc_bf16(64, DK, 0, 1), C / 16, dK, dKmn, sb + LY::T1,
                      sb + LY::T1L, sb + LY::KQW, 0, false);
            if constexpr (GDN)
                mma_split(tb + LY::cU, idesc_bf16(64, BV, 0, 1), C / 16, dK, dVT, sb + LY::T2,
                          sb + LY::T2L, sb + LY::V, 0, false);
        }
        if (!mma_done()) break;
#pragma unroll
        for (int c = 0; c < DK; c += 32) {  // Wk rows -> bf16 rows 2C..3C of the [K; Q; Wk] tile
            float x[32];
            tmem_ld32(taddr(tb, 32 * warp, LY::cWk + c), x);
            tmem_wait_ld();
            if (own_t) store32_split(sm + LY::KQW, nullptr, 2 * C + t_row, c, x, LY::KQW_BLK);
        }

        // ---- rank-L write terms: sum_l P_l U_l, O_w = sum_l Mqw_l U_l, F_w = sum_l W_l^T D U_l
        if (rank_l) {
            bool ok = true;
            for (int l = 0; l < L; ++l) {
                sync_for_mma();  // the previous MMAs have finished reading the l-tiles
                for (int e = tid; e < C * (DK / 8); e += NT) {
                    const int t = e / (DK / 8), ch = e % (DK / 8);
                    uint4 wv = make_uint4(0, 0, 0, 0);
                    if (t < n) {
                        const size_t g = ((((size_t)b * T + c0 + t) * H + h) * L + l) * DK + ch * 8;
                        wv = *reinterpret_cast<const uint4 *>(w + g);
                    }
                    st16(sm + LY::W, sw128_off(t, ch * 8, LY::W_BLK), wv);
                }
                for (int e = tid; e < C * (BV / 8); e += NT) {
                    const int t = e / (BV / 8), ch = e % (BV / 8);
                    uint4 uv = make_uint4(0, 0, 0, 0), dh = uv, dl = uv;
                    if (t < n) {
                        const size_t g = ((((size_t)b * T + c0 + t) * H + h) * L + l) * dv + v0 + ch * 8;
                        uv = *reinterpret_cast<const uint4 *>(u + g);
                        const __nv_bfloat16 *hv = reinterpret_cast<const __nv_bfloat16 *>(&uv);
                        float du[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) du[j] = sD[t] * __bfloat162float(hv[j]);
                        split8(du, dh, dl);
                    }
                    const uint32_t off = vt_off<BV>(t, ch * 8);
                    st16(sm + LY::V, off, uv);
                    st16(sm + LY::DU, off, dh);
                    st16(sm + LY::DUL, off, dl);
                }
                sync_for_mma();
                if (tid == 0)
                    mma_split(tb + LY::cG, idesc_bf16(128, C, 0, 0), DK / 16, dKQW,
                              [](uint32_t base, int ks) { return desc_k_sw128(base, ks, LY::W_BLK); },
                              sb + LY::KQW, 0, sb + LY::W, 0, false);
                if (!mma_done()) { ok = false; break; }
                {
                    const int t = (warp & 1) * 32 + lane;
                    const float gt = sG[t], bt = sBeta[t];
                    uint8_t *dh = sm + (warp < 2 ? LY::P : LY::MQW);
                    uint8_t *dl = sm + (warp < 2 ? LY::PL : LY::MQWL);
#pragma unroll
                    for (int c = 0; c < C; c += 32) {
                        float gr[32];
                        tmem_ld32(taddr(tb, 32 * warp, LY::cG + c), gr);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int i = c + j;
                            const bool keep = (warp < 2) ? (i < t) : (i <= t);
                            gr[j] = keep ? (warp < 2 ? bt : 1.f) * expf(gt - sG[i]) * gr[j] : 0.f;
                        }
                        store32_split(dh, dl, t, c, gr);
                    }
                }
                sync_for_mma();
                if (tid == 0) {
                    const bool acc = l > 0;
                    mma_split(tb + LY::cPU, idesc_bf16(64, BV, 0, 1), C / 16, dK, dVT, sb + LY::P,
                              sb + LY::PL, sb + LY::V, 0, acc);
                    mma_split(tb + LY::cO, idesc_bf16(64, BV, 0, 1), C / 16, dK, dVT, sb + LY::MQW,
                              sb + LY::MQWL, sb + LY::V, 0, acc);
                    mma_split(tb + LY::cDS, idesc_bf16(DK, BV, 1, 1), C / 16, dWmn, dVT, sb + LY::W,
                              0, sb + LY::DU, sb + LY::DUL, acc);
                }
                if (!mma_done()) { ok = false; break; }
            }
            if (!ok) break;
            {   // sum_l P_l U_l -> bf16 pair (B operand of X_u = T (sum_l P_l U_l))
                float x[BV];
                ld_row<BV>(tb, warp, LY::cPU, x);
                if (own_t) store_row_split<BV>(sm + LY::PU, sm + LY::PUL, t_row, x);
            }
            sync_for_mma();
            if (tid == 0)
                mma_split(tb + LY::cU, idesc_bf16(64, BV, 0, 1), C / 16, dK, dVT, sb + LY::T2,
                          sb + LY::T2L, sb + LY::PU, sb + LY::PUL, false);
            if (!mma_done()) break;
        }
        sync_for_mma();

        // ---- state-dependent: X_s = Wk S^T, QS = Q S^T
        if (tid == 0) {
            const uint32_t id = idesc_bf16(64, BV, 0, 1);
            mma_split(tb + LY::cXs, id, DK / 16, dKQW, dVT, sb + LY::KQW + 2 * C * 128, 0,
                      sb + LY::S, sb + LY::SL, false);
            mma_split(tb + LY::cQS, id, DK / 16, dKQW, dVT, sb + LY::KQW + C * 128, 0, sb + LY::S,
                      sb + LY::SL, false);
        }
        if (!mma_done()) break;
        {
            float xs[BV], uu[BV];
            ld_row<BV>(tb, warp, LY::cXs, xs);
            ld_row<BV>(tb, warp, LY::cU, uu);
            if (own_t) {
                float y[BV];
                const float dd = sD[t_row];
#pragma unroll
                for (int j = 0; j < BV; ++j)
                    y[j] = !wr ? -xs[j] : (GDN ? (uu[j] - xs[j]) : -(uu[j] + xs[j]));
                store_row_split<BV>(sm + LY::Y, sm + LY::YL, t_row, y);
#pragma unroll
                for (int j = 0; j < BV; ++j) y[j] *= dd;
                store_row_split<BV>(sm + LY::DY, sm + LY::DYL, t_row, y);
            }
        }
        sync_for_mma();
        // ---- O (+)= Mqk Y ; S'^T (+)= K^T D Y
        if (tid == 0) {
            mma_split(tb + LY::cO, idesc_bf16(64, BV, 0, 1), C / 16, dK, dVT, sb + LY::MQK,
                      sb + LY::MQKL, sb + LY::Y, sb + LY::YL, rank_l);
            mma_split(tb + LY::cDS, idesc_bf16(DK, BV, 1, 1), C / 16, dKmn, dVT, sb + LY::KQW, 0,
                      sb + LY::DY, sb + LY::DYL, rank_l);
        }
        if (!mma_done()) break;
        {
            float qs[BV], op[BV];
            ld_row<BV>(tb, warp, LY::cQS, qs);
            ld_row<BV>(tb, warp, LY::cO, op);
            if (own_t && t_row < n && !(p.flags & kNoOutput)) {
                const float gt = sGam[t_row];
                __nv_bfloat16 *dst = o + (((size_t)b * T + c0 + t_row) * H + h) * dv + v0;
#pragma unroll
                for (int c8 = 0; c8 < BV / 8; ++c8) {
                    uint4 pk;
                    pk.x = pack_bf16(fmaf(gt, qs[c8 * 8 + 0], op[c8 * 8 + 0]), fmaf(gt, qs[c8 * 8 + 1], op[c8 * 8 + 1]));
                    pk.y = pack_bf16(fmaf(gt, qs[c8 * 8 + 2], op[c8 * 8 + 2]), fmaf(gt, qs[c8 * 8 + 3], op[c8 * 8 + 3]));
                    pk.z = pack_bf16(fmaf(gt, qs[c8 * 8 + 4], op[c8 * 8 + 4]), fmaf(gt, qs[c8 * 8 + 5], op[c8 * 8 + 5]));
                    pk.w = pack_bf16(fmaf(gt, qs[c8 * 8 + 6], op[c8 * 8 + 6]), fmaf(gt, qs[c8 * 8 + 7], op[c8 * 8 + 7]));
                    *reinterpret_cast<uint4 *>(dst + c8 * 8) = pk;
                }
            }
            float ds[BV];
            ld_row<BV>(tb, warp, LY::cDS, ds);
            const float gC = expf(g_last);
            if (own_d) {
#pragma unroll
                for (int j = 0; j < BV; ++j) Sreg[j] = fmaf(gC, Sreg[j], ds[j]);
                store_row_split<BV>(sm + LY::S, sm + LY::SL, d_row, Sreg);
            }
        }
        sync_for_mma();
    }

    if (p.S_final && own_d && failed_sh == 0) {
#pragma unroll
        for (int j = 0; j < BV; ++j) p.S_final[(head * dv + v0 + j) * DK + d_row] = Sreg[j];
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, TMEM_COLS);
}

template <int DK, int BV, bool GDN>
cudaError_t launch_tc(const ScanArgs &a, cudaStream_t s) {
    using LY = TcLayout<DK, BV, GDN>;
    // at least ~116 KB so that a single CTA (holding all 512 TMEM columns) runs per SM
    constexpr size_t bytes = LY::BYTES < 120 * 1024 ? 120 * 1024 : LY::BYTES;
    static_assert(bytes <= 227 * 1024, "shared memory budget");
    auto kern = scan_tc_kernel<DK, BV, GDN>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (err != cudaSuccess) return err;
    dim3 grid(a.dv / BV, a.H, a.B);
    launch_probe_mark(s);
    kern<<<grid, NT, bytes, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

// Shapes the tensor-core path takes: bf16 I/O, dk == dv in {64, 128}, L <= 8.
bool scan_tc_supported(const ScanArgs &a, bool io_f32) {
    return !io_f32 && a.dk == a.dv && (a.dk == 64 || a.dk == 128) && a.L <= 8;
}

cudaError_t launch_scan_tc(const ScanArgs &a, cudaStream_t s) {
    const bool gdn = (a.u == nullptr);
    if (a.dk == 128) {
        return gdn ? launch_tc<128, 32, true>(a, s) : launch_tc<128, 32, false>(a, s);
    }
    return gdn ? launch_tc<64, 64, true>(a, s) : launch_tc<64, 64, false>(a, s);
}

}  // namespace prism
