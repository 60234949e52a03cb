// scan_gdn.cu -- the Gated-DeltaNet write (u = beta v, w = k) as two tensor-core kernels.
//
// The chunk form (see scan_tc.cu) splits each chunk's work into a state-independent part and a
// state-dependent part.  The first depends only on the chunk's own tokens, so it runs for every
// (batch, head, chunk) at once in `gdn_prep_kernel`, once per head (not once per value slice):
//   G = [K; Q] K^T,   A = strict(diag(beta) Gamma o K K^T),   Mqk = incl(Gamma o Q K^T),
//   T = (I + A)^{-1},  Wk = T diag(beta e^g) K,  and the operand T diag(beta) of U = T diag(beta) V.
// It writes Wk (bf16), T diag(beta) and Mqk (bf16 hi/lo pairs) and g to a per-chunk record in the
// workspace, already laid out as the 128B-swizzled shared-memory images the MMAs read.
// `gdn_state_kernel` then walks the chunks of one (batch, head, value slice) in order with the
// fp32 state on chip; per chunk it prefetches the next chunk's tiles (cp.async, double buffered)
// and runs only two dependent MMA rounds:
//   U = T diag(beta) V,  X_s = Wk S^T,  QS = Q S^T;   Y = U - X_s
//   O = diag(e^g) QS + Mqk Y,   S'^T = e^{g_n} S^T + K^T D Y.
// ("Sequential Parallel Duality in Prefix Scannable Models", method overview: encode all chunks
// in parallel, then combine them in order; banbantang.com PRISM article, section 1(4): the GDN
// forget and rank-1 write.)  Prep runs over chunks last-first, so the records the state kernel
// needs first are the ones most recently written and most likely still in L2.

#include "chunk_common.cuh"

namespace prism {
namespace {

constexpr int NT = 128;

// One workspace record per (b, h, chunk): swizzled shared-memory images.
template <int DK>
struct GdnRec {
    static constexpr uint32_t WK_BLK = C * 128;                  // 64 rows x 128 B per 64 columns
    static constexpr uint32_t WK = 0;                             // Wk, bf16
    static constexpr uint32_t T2 = WK + WK_BLK * (DK / 64);       // T diag(beta), hi then lo
    static constexpr uint32_t T2L = T2 + C * 128;
    static constexpr uint32_t MQK = T2L + C * 128;                // Mqk, hi then lo
    static constexpr uint32_t MQKL = MQK + C * 128;
    static constexpr uint32_t G = MQKL + C * 128;                 // g_t, 64 floats
    static constexpr uint32_t BYTES = G + 1024;
};
constexpr size_t kRecOffset = 1024;  // records start after the status block

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)),
                 "l"(gsrc), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// ------------------------------------------------------------------------------------------------
// prep: one CTA per (chunk, head, batch)

template <int DK>
struct PrepLayout {
    static constexpr uint32_t KQ_BLK = 2 * C * 128;     // [K; Q] rows of one 64-column block
    static constexpr uint32_t KQ = 0;
    static constexpr uint32_t T1 = KQ + KQ_BLK * (DK / 64);
    static constexpr uint32_t T1L = T1 + C * 128;
    static constexpr uint32_t AF = T1L + C * 128;       // fp32 A, solved in place into T
    static constexpr uint32_t TMP = AF + C * AS * 4;
    static constexpr uint32_t GATES = TMP + 32 * 33 * 4;
    static constexpr uint32_t BYTES = GATES + 3 * C * 4 + 1024;
};

template <int DK>
__global__ void __launch_bounds__(NT) gdn_prep_kernel(ScanArgs p, uint8_t *ws, int nch) {
    using LY = PrepLayout<DK>;
    using RC = GdnRec<DK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t mma_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int failed_sh;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = nch - 1 - blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int H = p.H, T = p.T;
    const int c0 = c * C, n = min(C, T - c0);
    const __nv_bfloat16 *q = (const __nv_bfloat16 *)p.q, *k = (const __nv_bfloat16 *)p.k;
    uint8_t *rec = ws + kRecOffset + (((size_t)b * H + h) * nch + c) * RC::BYTES;
    float *sA = (float *)(sm + LY::AF);
    float *sTmp = (float *)(sm + LY::TMP);
    float *sG = (float *)(sm + LY::GATES);
    float *sBeta = sG + C;
    float *sGam = sBeta + C;
    const uint32_t sb = smem_u32(sm);

    // K and Q rows (zero rows past the end of the sequence are identity tokens)
    for (int e = tid; e < C * (DK / 8); e += NT) {
        const int t = e / (DK / 8), ch = e % (DK / 8);
        const bool ok = t < n;
        const size_t g = ok ? ((((size_t)b * T + c0 + t) * H + h) * DK + ch * 8) : 0;
        cp_async16(sm + LY::KQ + sw128_off(t, ch * 8, LY::KQ_BLK), k + g, ok ? 16 : 0);
        cp_async16(sm + LY::KQ + sw128_off(C + t, ch * 8, LY::KQ_BLK), q + g, ok ? 16 : 0);
    }
    cp_async_commit();
    if (warp == 0) tmem_alloc(&tmem_base_sh, 128);
    if (tid == 0) {
        mbar_init(&mma_bar, 1);
        mbar_fence_init();
        failed_sh = 0;
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
    cp_async_wait<0>();
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tb = tmem_base_sh;
    if (tid < C) {
        sGam[tid] = expf(sG[tid]);
        reinterpret_cast<float *>(rec + RC::G)[tid] = sG[tid];
    }

    // G = [K; Q] K^T
    if (tid == 0)
        mma_split(tb, idesc_bf16(128, C, 0, 0), DK / 16,
                  [](uint32_t base, int ks) { return desc_k_sw128(base, ks, LY::KQ_BLK); },
                  [](uint32_t base, int ks) { return desc_k_sw128(base, ks, LY::KQ_BLK); },
                  sb + LY::KQ, 0, sb + LY::KQ, 0, false);
    if (tid == 0) mma_commit(&mma_bar);
    __syncwarp();
    if (!mbar_wait(&mma_bar, 0, p.status)) failed_sh = 1;
    fence_after_sync();
    __syncthreads();
    bool ok = failed_sh == 0;  // uniform across the CTA
    if (ok) {
        const int t = (warp & 1) * 32 + lane;
        const float gt = sG[t], bt = sBeta[t];
#pragma unroll
        for (int cc = 0; cc < C; cc += 32) {
            float gr[32];
            tmem_ld32(taddr(tb, 32 * warp, cc), gr);
            tmem_wait_ld();
            if (warp < 2) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int i = cc + j;
                    sA[t * AS + i] = (i < t) ? bt * expf(gt - sG[i]) * gr[j] : 0.f;
                }
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int i = cc + j;
                    gr[j] = (i <= t) ? expf(gt - sG[i]) * gr[j] : 0.f;
                }
                store32_split(rec + RC::MQK, rec + RC::MQKL, t, cc, gr);
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (ok) {
        solve_unit_lower<NT>(sA, sA, sTmp, tid);
        for (int e = tid; e < C * (C / 8); e += NT) {
            const int t = e / (C / 8), c8 = e % (C / 8);
            float a1[8], a2[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = c8 * 8 + j;
                const float tv = (i <= t) ? sA[t * AS + i] : 0.f;
                a1[j] = tv * sBeta[i] * sGam[i];
                a2[j] = tv * sBeta[i];
            }
            uint4 h1, l1, h2, l2;
            split8(a1, h1, l1);
            split8(a2, h2, l2);
            const uint32_t off = sw128_off(t, c8 * 8, 0);
            st16(sm + LY::T1, off, h1);
            st16(sm + LY::T1L, off, l1);
            st16(rec + RC::T2, off, h2);
            st16(rec + RC::T2L, off, l2);
        }
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    // Wk = T diag(beta gamma) K  (M = 64, N = DK; K read as an MN-major operand)
    if (ok && tid == 0) {
        mma_split(tb, idesc_bf16(64, DK, 0, 1), C / 16,
                  [](uint32_t base, int ks) { return desc_k_sw128(base, ks, 0); },
                  [](uint32_t base, int ks) { return desc_mn_sw128(base, ks, LY::KQ_BLK); },
                  sb + LY::T1, sb + LY::T1L, sb + LY::KQ, 0, false);
        mma_commit(&mma_bar);
    }
    __syncwarp();
    if (ok && !mbar_wait(&mma_bar, 1, p.status)) failed_sh = 1;
    fence_after_sync();
    __syncthreads();
    ok = failed_sh == 0;
    if (ok) {
        const bool own_t = lane < 16;
        const int t_row = 16 * warp + lane;
#pragma unroll
        for (int cc = 0; cc < DK; cc += 32) {
            float x[32];
            tmem_ld32(taddr(tb, 32 * warp, cc), x);
            tmem_wait_ld();
            if (own_t) store32_split(rec + RC::WK, nullptr, t_row, cc, x, RC::WK_BLK);
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 128);
}

// ------------------------------------------------------------------------------------------------
// state: one CTA per (value slice, head, batch), chunks in order

template <int DK, int BV>
struct StateLayout {
    static constexpr uint32_t KQW_BLK = 3 * C * 128;      // [K; Q; Wk] rows of one 64-col block
    static constexpr uint32_t ROWB = (BV == 32) ? 64 : 128;
    static constexpr uint32_t VT = C * ROWB;
    // one buffer of chunk inputs
    static constexpr uint32_t B_KQW = 0;
    static constexpr uint32_t B_V = B_KQW + KQW_BLK * (DK / 64);
    static constexpr uint32_t B_T2 = B_V + VT;             // T diag(beta) hi, lo (contiguous)
    static constexpr uint32_t B_T2L = B_T2 + C * 128;
    static constexpr uint32_t B_MQK = B_T2L + C * 128;     // Mqk hi, lo
    static constexpr uint32_t B_MQKL = B_MQK + C * 128;
    static constexpr uint32_t B_G = B_MQKL + C * 128;      // g (64 floats)
    static constexpr uint32_t BUF = B_G + 1024;
    // state-only tiles
    static constexpr uint32_t S = 2 * BUF;
    static constexpr uint32_t SL = S + DK * ROWB;
    static constexpr uint32_t Y = SL + DK * ROWB;
    static constexpr uint32_t YL = Y + VT;
    static constexpr uint32_t DY = YL + VT;
    static constexpr uint32_t DYL = DY + VT;
    static constexpr uint32_t GATES = DYL + VT;             // gamma, D: 2 x C floats
    static constexpr uint32_t BYTES = GATES + 2 * C * 4 + 1024;
    // TMEM columns
    static constexpr uint32_t cU = 0, cXs = BV, cQS = 2 * BV, cO = 3 * BV, cDS = 4 * BV;
    static constexpr uint32_t TCOLS = (5 * BV <= 128) ? 128 : (5 * BV <= 256 ? 256 : 512);
};

template <int DK, int BV>
__device__ __forceinline__ void state_issue_loads(const ScanArgs &p, const uint8_t *ws, int nch,
                                                  int c, uint8_t *buf, int tid) {
    using LY = StateLayout<DK, BV>;
    using RC = GdnRec<DK>;
    const int v0 = blockIdx.x * BV, h = blockIdx.y, b = blockIdx.z;
    const int H = p.H, T = p.T, dv = p.dv;
    const int c0 = c * C, n = min(C, T - c0);
    const __nv_bfloat16 *q = (const __nv_bfloat16 *)p.q, *k = (const __nv_bfloat16 *)p.k;
    const __nv_bfloat16 *v = (const __nv_bfloat16 *)p.v;
    for (int e = tid; e < C * (DK / 8); e += NT) {
        const int t = e / (DK / 8), ch = e % (DK / 8);
        const bool ok = t < n;
        const size_t g = ok ? ((((size_t)b * T + c0 + t) * H + h) * DK + ch * 8) : 0;
        cp_async16(buf + LY::B_KQW + sw128_off(t, ch * 8, LY::KQW_BLK), k + g, ok ? 16 : 0);
        cp_async16(buf + LY::B_KQW + sw128_off(C + t, ch * 8, LY::KQW_BLK), q + g, ok ? 16 : 0);
    }
    for (int e = tid; e < C * (BV / 8); e += NT) {
        const int t = e / (BV / 8), ch = e % (BV / 8);
        const bool ok = t < n;
        const size_t g = ok ? ((((size_t)b * T + c0 + t) * H + h) * dv + v0 + ch * 8) : 0;
        cp_async16(buf + LY::B_V + vt_off<BV>(t, ch * 8), v + g, ok ? 16 : 0);
    }
    const uint8_t *rec = ws + kRecOffset + (((size_t)b * H + h) * nch + c) * RC::BYTES;
    // Wk image: 64-column blocks land in rows 2C..3C of the stacked tile (swizzle preserved:
    // both bases are 1024-aligned and 2C is a multiple of 8)
    for (int e = tid; e < (DK / 64) * (RC::WK_BLK / 16); e += NT) {
        const int blk = e / (RC::WK_BLK / 16), off = (e % (RC::WK_BLK / 16)) * 16;
        cp_async16(buf + LY::B_KQW + blk * LY::KQW_BLK + 2 * C * 128 + off,
                   rec + RC::WK + blk * RC::WK_BLK + off, 16);
    }
    // T diag(beta) pair, Mqk pair, g: contiguous in the record and in the buffer
    for (int e = tid; e < (4 * C * 128 + C * 4) / 16; e += NT)
        cp_async16(buf + LY::B_T2 + e * 16, rec + RC::T2 + e * 16, 16);
}

template <int DK, int BV>
__global__ void __launch_bounds__(NT, 1) gdn_state_kernel(ScanArgs p, const uint8_t *ws, int nch) {
    using LY = StateLayout<DK, BV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t mma_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int failed_sh;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int v0 = blockIdx.x * BV, h = blockIdx.y, b = blockIdx.z;
    const int H = p.H, T = p.T, dv = p.dv;
    __nv_bfloat16 *o = (__nv_bfloat16 *)p.o;
    const size_t head = (size_t)b * H + h;
    float *sGam = (float *)(sm + LY::GATES);
    float *sD = sGam + C;
    const uint32_t sb = smem_u32(sm);

    if (nch > 0) state_issue_loads<DK, BV>(p, ws, nch, 0, sm, tid);
    cp_async_commit();
    if (warp == 0) tmem_alloc(&tmem_base_sh, LY::TCOLS);
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
    auto dK = [](uint32_t base, int ks) { return desc_k_sw128(base, ks, 0); };
    auto dKQW = [](uint32_t base, int ks) { return desc_k_sw128(base, ks, LY::KQW_BLK); };
    auto dKmn = [](uint32_t base, int ks) { return desc_mn_sw128(base, ks, LY::KQW_BLK); };
    auto dVT = [](uint32_t base, int ks) { return desc_vt<BV>(base, ks); };

    const bool own_d = (DK == 128) ? true : (lane < 16);
    const int d_row = (DK == 128) ? tid : (16 * warp + lane);
    float Sreg[BV];
#pragma unroll
    for (int j = 0; j < BV; ++j) Sreg[j] = 0.f;
    if (own_d && p.S0) {
#pragma unroll
        for (int j = 0; j < BV; ++j) Sreg[j] = p.S0[(head * dv + v0 + j) * DK + d_row];
    }
    if (own_d) store_row_split<BV>(sm + LY::S, sm + LY::SL, d_row, Sreg);
    const bool own_t = lane < 16;
    const int t_row = 16 * warp + lane;

    for (int c = 0; c < nch; ++c) {
        const int c0 = c * C, n = min(C, T - c0);
        uint8_t *buf = sm + (c & 1) * LY::BUF;
        const uint32_t bb = sb + (c & 1) * LY::BUF;
        if (c + 1 < nch) state_issue_loads<DK, BV>(p, ws, nch, c + 1, sm + ((c + 1) & 1) * LY::BUF, tid);
        cp_async_commit();
        cp_async_wait<1>();  // this chunk's group has landed; the next chunk's stays in flight
        const float *g = reinterpret_cast<const float *>(buf + LY::B_G);
        __syncthreads();
        const float g_last = g[C - 1];
        if (tid < C) {
            sGam[tid] = expf(g[tid]);
            sD[tid] = tid < n ? expf(g_last - g[tid]) : 0.f;
        }
        sync_for_mma();

        // U = T diag(beta) V ;  X_s = Wk S^T ;  QS = Q S^T
        if (tid == 0) {
            const uint32_t id = idesc_bf16(64, BV, 0, 1);
            mma_split(tb + LY::cU, id, C / 16, dK, dVT, bb + LY::B_T2, bb + LY::B_T2L, bb + LY::B_V, 0, false);
            mma_split(tb + LY::cXs, id, DK / 16, dKQW, dVT, bb + LY::B_KQW + 2 * C * 128, 0,
                      sb + LY::S, sb + LY::SL, false);
            mma_split(tb + LY::cQS, id, DK / 16, dKQW, dVT, bb + LY::B_KQW + C * 128, 0,
                      sb + LY::S, sb + LY::SL, false);
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
                for (int j = 0; j < BV; ++j) y[j] = uu[j] - xs[j];
                store_row_split<BV>(sm + LY::Y, sm + LY::YL, t_row, y);
#pragma unroll
                for (int j = 0; j < BV; ++j) y[j] *= dd;
                store_row_split<BV>(sm + LY::DY, sm + LY::DYL, t_row, y);
            }
        }
        sync_for_mma();
        // O = Mqk Y ;  S'^T contribution K^T D Y
        if (tid == 0) {
            mma_split(tb + LY::cO, idesc_bf16(64, BV, 0, 1), C / 16, dK, dVT, bb + LY::B_MQK,
                      bb + LY::B_MQKL, sb + LY::Y, sb + LY::YL, false);
            mma_split(tb + LY::cDS, idesc_bf16(DK, BV, 1, 1), C / 16, dKmn, dVT, bb + LY::B_KQW, 0,
                      sb + LY::DY, sb + LY::DYL, false);
        }
        if (!mma_done()) break;
        {
            float qs[BV], op[BV];
            ld_row<BV>(tb, warp, LY::cQS, qs);
            ld_row<BV>(tb, warp, LY::cO, op);
            if (own_t && t_row < n) {
                const float gt = sGam[t_row];
                __nv_bfloat16 *dst = o + (((size_t)b * T + c0 + t_row) * H + h) * dv + v0;
#pragma unroll
                for (int c8 = 0; c8 < BV / 8; ++c8) {
                    float r[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) r[j] = fmaf(gt, qs[c8 * 8 + j], op[c8 * 8 + j]);
                    uint4 pk;
                    pk.x = pack_bf16(r[0], r[1]);
                    pk.y = pack_bf16(r[2], r[3]);
                    pk.z = pack_bf16(r[4], r[5]);
                    pk.w = pack_bf16(r[6], r[7]);
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
    cp_async_wait<0>();

    if (p.S_final && own_d && failed_sh == 0) {
#pragma unroll
        for (int j = 0; j < BV; ++j) p.S_final[(head * dv + v0 + j) * DK + d_row] = Sreg[j];
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, LY::TCOLS);
}

template <int DK, int BV>
cudaError_t launch_gdn(const ScanArgs &a, void *ws, cudaStream_t s) {
    const int nch = (a.T + C - 1) / C;
    {
        using LY = PrepLayout<DK>;
        auto kern = gdn_prep_kernel<DK>;
        cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)LY::BYTES);
        if (err != cudaSuccess) return err;
        if (nch > 0) {
            dim3 grid(nch, a.H, a.B);
            kern<<<grid, NT, LY::BYTES, s>>>(a, (uint8_t *)ws, nch);
            err = cudaGetLastError();
            if (err != cudaSuccess) return err;
        }
    }
    {
        using LY = StateLayout<DK, BV>;
        static_assert(LY::BYTES <= 227 * 1024, "shared memory budget");
        auto kern = gdn_state_kernel<DK, BV>;
        cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)LY::BYTES);
        if (err != cudaSuccess) return err;
        dim3 grid(a.dv / BV, a.H, a.B);
        kern<<<grid, NT, LY::BYTES, s>>>(a, (const uint8_t *)ws, nch);
        return cudaGetLastError();
    }
}

}  // namespace

// Workspace bytes of the two-kernel GDN path: the status block plus one record per chunk.
size_t gdn_workspace_bytes(int B, int H, int T, int dk) {
    const size_t nch = (size_t)((T + C - 1) / C);
    const size_t rec = dk == 128 ? GdnRec<128>::BYTES : GdnRec<64>::BYTES;
    return kRecOffset + (size_t)B * H * nch * rec;
}

cudaError_t launch_scan_gdn(const ScanArgs &a, void *ws, cudaStream_t s) {
    if (a.dk == 128) return launch_gdn<128, 32>(a, ws, s);
    return launch_gdn<64, 64>(a, ws, s);
}

}  // namespace prism
