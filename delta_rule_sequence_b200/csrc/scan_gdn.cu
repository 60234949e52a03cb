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
// fp32 state on chip; per chunk it prefetches the next chunk's tiles (TMA, double buffered)
// and runs only two dependent MMA rounds:
//   U = T diag(beta) V,  X_s = Wk S^T,  QS = Q S^T;   Y = U - X_s
//   O = diag(e^g) QS + Mqk Y,   S'^T = e^{g_n} S^T + K^T D Y.
// ("Sequential Parallel Duality in Prefix Scannable Models", method overview: encode all chunks
// in parallel, then combine them in order; banbantang.com PRISM article, section 1(4): the GDN
// forget and rank-1 write.)  Prep runs over chunks last-first, so the records the state kernel
// needs first are the ones most recently written and most likely still in L2.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "chunk_common.cuh"

namespace prism {
namespace {

constexpr int NT = 128;

// TMA descriptors of the bf16 activations, viewed as 4-D {d, H, T, B} (innermost first) so that
// a box {64 | BV, 1, 64, 1} is one head's chunk; rows past T read as zeros.
struct GdnMaps {
    CUtensorMap k, q, v;
};

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
__global__ void __launch_bounds__(NT) gdn_prep_kernel(ScanArgs p, const __grid_constant__ GdnMaps maps,
                                                     uint8_t *ws, int nch) {
    using LY = PrepLayout<DK>;
    using RC = GdnRec<DK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t mma_bar, ld_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int failed_sh;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = nch - 1 - blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int H = p.H, T = p.T;
    const int c0 = c * C, n = min(C, T - c0);
    uint8_t *rec = ws + kRecOffset + (((size_t)b * H + h) * nch + c) * RC::BYTES;
    float *sA = (float *)(sm + LY::AF);
    float *sTmp = (float *)(sm + LY::TMP);
    float *sG = (float *)(sm + LY::GATES);
    float *sBeta = sG + C;
    float *sGam = sBeta + C;
    const uint32_t sb = smem_u32(sm);

    // K and Q boxes by TMA (rows past the end of the sequence arrive as zeros: identity tokens)
    if (tid == 0) {
        mbar_init(&mma_bar, 1);
        mbar_init(&ld_bar, 1);
        mbar_fence_init();
        failed_sh = 0;
        mbar_expect_tx(&ld_bar, 2 * (DK / 64) * C * 128);
        for (int blk = 0; blk < DK / 64; ++blk) {
            tma_load_4d(sm + LY::KQ + blk * LY::KQ_BLK, &maps.k, blk * 64, h, c0, b, &ld_bar);
            tma_load_4d(sm + LY::KQ + blk * LY::KQ_BLK + C * 128, &maps.q, blk * 64, h, c0, b, &ld_bar);
        }
    }
    if (warp == 0) tmem_alloc(&tmem_base_sh, 128);
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
    if (!mbar_wait(&ld_bar, 0, p.status)) failed_sh = 1;
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tb = tmem_base_sh;
    if (tid < C) {
        sGam[tid] = expf(sG[tid]);
        reinterpret_cast<float *>(rec + RC::G)[tid] = sG[tid];
    }

    // G = [K; Q] K^T
    auto okq = [](int ks) { return (uint64_t)koff_k_sw128(ks, LY::KQ_BLK); };
    auto ok0 = [](int ks) { return (uint64_t)koff_k_sw128(ks, 0); };
    auto omn = [](int ks) { return (uint64_t)koff_mn_sw128(ks); };
    if (tid == 0 && failed_sh == 0) {
        const uint64_t dkq = make_desc(sb + LY::KQ, 16, 1024, 2);
        mma_steps<DK / 16>(tb, idesc_bf16(128, C, 0, 0), dkq, dkq, okq, okq, false);
    }
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
                    sA[t * AS + i] = (i < t) ? bt * __expf(gt - sG[i]) * gr[j] : 0.f;
                }
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int i = cc + j;
                    gr[j] = (i <= t) ? __expf(gt - sG[i]) * gr[j] : 0.f;
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
        const uint32_t id = idesc_bf16(64, DK, 0, 1);
        const uint64_t dK = make_desc(sb + LY::KQ, LY::KQ_BLK, 1024, 2);
        mma_steps<C / 16>(tb, id, make_desc(sb + LY::T1, 16, 1024, 2), dK, ok0, omn, false);
        mma_steps<C / 16>(tb, id, make_desc(sb + LY::T1L, 16, 1024, 2), dK, ok0, omn, true);
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
//
// Two MMA rounds per chunk, shaped to keep the tcgen05 instruction count low:
//   round 1:  D1  = [Q; Wk] [S_hi | S_lo]                  (M = 128, N = 2 BV: QS and X_s, hi and lo
//                                                           halves side by side)
//             D1[:, :BV] -= [0; T2_hi] V + [0; T2_lo] V    (U lands in the X_s rows; zero tile on top)
//   round 2:  D3  = [Mqk_hi; 0] [Y_hi | Y_lo] ;  D3[:, :BV] += [Mqk_lo; 0] Y_hi
//             D4  = K^T [DY_hi | DY_lo]
// so that every operand row t of the chunk sits in TMEM lane t (QS, O) or lane 64 + t (X_s - U).
// K, Q and V arrive by TMA tiled loads, the per-chunk records (Wk, T2, Mqk, g) by bulk copies.

template <int DK, int BV>
struct StateLayout {
    static constexpr uint32_t KQW_BLK = 3 * C * 128;      // [K; Q; Wk] rows of one 64-col block
    static constexpr uint32_t ROWB = (BV == 32) ? 64 : 128;
    static constexpr uint32_t VT = C * ROWB;              // C x BV tile (V slice)
    static constexpr int N2 = 2 * BV;                     // hi | lo side by side
    // double-buffered chunk inputs
    static constexpr uint32_t B_KQW = 0;
    static constexpr uint32_t B_V = B_KQW + KQW_BLK * (DK / 64);
    static constexpr uint32_t B_G = B_V + VT;               // g (64 floats)
    static constexpr uint32_t BUF = B_G + 1024;
    // single-buffered operands: [Mqk_hi][0][T2_hi][Mqk_lo][0][T2_lo]
    static constexpr uint32_t MH = 2 * BUF;
    static constexpr uint32_t Z1 = MH + C * 128;
    static constexpr uint32_t T2H = Z1 + C * 128;
    static constexpr uint32_t ML = T2H + C * 128;
    static constexpr uint32_t Z2 = ML + C * 128;
    static constexpr uint32_t T2L = Z2 + C * 128;
    // S^T [d][hi | lo], Y [t][hi | lo], D Y [t][hi | lo]: MN-major, 64-column blocks
    static constexpr uint32_t S_BLK = DK * 128;
    static constexpr uint32_t S = T2L + C * 128;
    static constexpr uint32_t Y_BLK = C * 128;
    static constexpr uint32_t Y = S + S_BLK * (N2 / 64);
    static constexpr uint32_t DY = Y + Y_BLK * (N2 / 64);
    static constexpr uint32_t GATES = DY + Y_BLK * (N2 / 64);  // gamma, D: 2 x C floats
    static constexpr uint32_t BYTES = GATES + 2 * C * 4 + 1024;
    // TMEM columns
    static constexpr uint32_t cD1 = 0, cD3 = N2, cD4 = 2 * N2, cU = 3 * N2;
    static constexpr uint32_t TCOLS = (3 * N2 + BV <= 128) ? 128 : (3 * N2 + BV <= 256 ? 256 : 512);
};

// An N2-wide row of fp32 (hi | lo of one value each) stored as bf16 into an MN-major tile of
// 64-column 128B-swizzled blocks: cols [0, BV) get bf16(x), cols [BV, 2BV) get bf16(x - hi).
template <int BV>
__device__ __forceinline__ void store_row_pair(uint8_t *tile, uint32_t blk_bytes, int row,
                                               const float *x) {
#pragma unroll
    for (int c8 = 0; c8 < BV / 8; ++c8) {
        uint4 h, l;
        split8(x + c8 * 8, h, l);
        st16(tile, sw128_off(row, c8 * 8, blk_bytes), h);
        st16(tile, sw128_off(row, BV + c8 * 8, blk_bytes), l);
    }
}

// out[j] = D[lane row][col + j] + D[lane row][col + BV + j]: the hi and lo halves of a pair MMA.
template <int BV>
__device__ __forceinline__ void ld_pair_sum(uint32_t tbase, int warp, uint32_t col, float *out) {
#pragma unroll
    for (int c = 0; c < BV; c += 32) {
        float a[32], b[32];
        tmem_ld32(taddr(tbase, 32 * warp, col + c), a);
        tmem_ld32(taddr(tbase, 32 * warp, col + BV + c), b);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) out[c + j] = a[j] + b[j];
    }
}

template <int DK>
__device__ __forceinline__ const uint8_t *record(const ScanArgs &p, const uint8_t *ws, int nch, int c) {
    return ws + kRecOffset + (((size_t)blockIdx.z * p.H + blockIdx.y) * nch + c) * GdnRec<DK>::BYTES;
}

// Warp roles of the state kernel: warps 0-3 epilogue (TMEM lane quarters 0-3), warp 4 issues the
// MMAs, warp 5 issues the loads.  Every hand-off is an mbarrier; every wait is bounded.
constexpr int ST_THREADS = 192;
constexpr int EPI_THREADS = 128;

struct StateBars {
    uint64_t full[2];      // chunk inputs landed (tx): K, Q, V, Wk, g
    uint64_t empty[2];     // chunk buffer released: last MMA reading it (commit) + epilogue (g read)
    uint64_t t2_full, t2_empty, mq_full, mq_empty;
    uint64_t s_ready, y_ready;      // epilogue -> MMA: S^T tile, Y / DY tiles written
    uint64_t d1_full, d4_full, d3_full;  // MMA -> epilogue: accumulators complete
};

template <int DK, int BV>
__global__ void __launch_bounds__(ST_THREADS, 1) gdn_state_kernel(ScanArgs p,
                                                                 const __grid_constant__ GdnMaps maps,
                                                                 const uint8_t *ws, int nch) {
    using LY = StateLayout<DK, BV>;
    using RC = GdnRec<DK>;
    constexpr int N2 = LY::N2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ StateBars bars;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int failed_sh;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int v0 = blockIdx.x * BV, h = blockIdx.y, b = blockIdx.z;
    const int H = p.H, T = p.T, dv = p.dv;
    const size_t head = (size_t)b * H + h;
    const uint32_t sb = smem_u32(sm);

    if (warp == 0) tmem_alloc(&tmem_base_sh, LY::TCOLS);
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars.full[i], 1);
            mbar_init(&bars.empty[i], 2);
        }
        mbar_init(&bars.t2_full, 1);
        mbar_init(&bars.t2_empty, 1);
        mbar_init(&bars.mq_full, 1);
        mbar_init(&bars.mq_empty, 1);
        mbar_init(&bars.s_ready, 1);
        mbar_init(&bars.y_ready, 1);
        mbar_init(&bars.d1_full, 1);
        mbar_init(&bars.d4_full, 1);
        mbar_init(&bars.d3_full, 1);
        mbar_fence_init();
        failed_sh = 0;
    }
    for (int e = tid; e < C * 128 / 16; e += ST_THREADS) {  // zero tiles under Mqk and over T2
        st16(sm + LY::Z1, e * 16, make_uint4(0, 0, 0, 0));
        st16(sm + LY::Z2, e * 16, make_uint4(0, 0, 0, 0));
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tb = tmem_base_sh;
    uint32_t *status = p.status;
    auto fail = [&]() { failed_sh = 1; };
    auto failed = [&]() { return *(volatile int *)&failed_sh != 0; };

    if (warp == 5) {
        // ---------------- loads ----------------
        if (lane == 0) {
            auto load_chunk = [&](int c) {
                const uint8_t *rec = record<DK>(p, ws, nch, c);
                uint8_t *buf = sm + (c & 1) * LY::BUF;
                uint64_t *bar = &bars.full[c & 1];
                const int c0 = c * C;
                mbar_expect_tx(bar, 2 * (DK / 64) * C * 128 + LY::VT + (DK / 64) * RC::WK_BLK + C * 4);
                for (int blk = 0; blk < DK / 64; ++blk) {
                    uint8_t *dst = buf + LY::B_KQW + blk * LY::KQW_BLK;
                    tma_load_4d(dst, &maps.k, blk * 64, h, c0, b, bar);
                    tma_load_4d(dst + C * 128, &maps.q, blk * 64, h, c0, b, bar);
                    bulk_g2s(dst + 2 * C * 128, rec + RC::WK + blk * RC::WK_BLK, RC::WK_BLK, bar);
                }
                tma_load_4d(buf + LY::B_V, &maps.v, v0, h, c0, b, bar);
                bulk_g2s(buf + LY::B_G, rec + RC::G, C * 4, bar);
            };
            for (int c = 0; c < nch && !failed(); ++c) {
                const uint8_t *rec = record<DK>(p, ws, nch, c);
                if (c >= 2 && !mbar_wait(&bars.empty[c & 1], ((c - 2) >> 1) & 1, status)) { fail(); break; }
                load_chunk(c);
                if (c >= 1 && !mbar_wait(&bars.t2_empty, (c - 1) & 1, status)) { fail(); break; }
                mbar_expect_tx(&bars.t2_full, 2 * C * 128);
                bulk_g2s(sm + LY::T2H, rec + RC::T2, C * 128, &bars.t2_full);
                bulk_g2s(sm + LY::T2L, rec + RC::T2L, C * 128, &bars.t2_full);
                if (c >= 1 && !mbar_wait(&bars.mq_empty, (c - 1) & 1, status)) { fail(); break; }
                mbar_expect_tx(&bars.mq_full, 2 * C * 128);
                bulk_g2s(sm + LY::MH, rec + RC::MQK, C * 128, &bars.mq_full);
                bulk_g2s(sm + LY::ML, rec + RC::MQKL, C * 128, &bars.mq_full);
            }
        }
    } else if (warp == 4) {
        // ---------------- MMA issue ----------------
        if (lane == 0) {
            auto oKQW = [](int ks) { return (uint64_t)koff_k_sw128(ks, LY::KQW_BLK); };
            auto oK0 = [](int ks) { return (uint64_t)koff_k_sw128(ks, 0); };
            auto oMN = [](int ks) { return (uint64_t)koff_mn_sw128(ks); };
            auto oVT = [](int ks) { return (uint64_t)(BV == 32 ? koff_mn_sw64(ks) : koff_mn_sw128(ks)); };
            const uint64_t dS2 = make_desc(sb + LY::S, LY::S_BLK, 1024, 2);
            const uint64_t dY2 = make_desc(sb + LY::Y, LY::Y_BLK, 1024, 2);
            const uint64_t dDY2 = make_desc(sb + LY::DY, LY::Y_BLK, 1024, 2);
            const uint64_t dZ1 = make_desc(sb + LY::Z1, 16, 1024, 2), dZ2 = make_desc(sb + LY::Z2, 16, 1024, 2);
            const uint64_t dMH = make_desc(sb + LY::MH, 16, 1024, 2), dML = make_desc(sb + LY::ML, 16, 1024, 2);
            const uint32_t idU = idesc_bf16(128, BV, 0, 1) | (1u << 13);  // negated A
            const uint32_t idS = idesc_bf16(128, N2, 0, 1);
            for (int c = 0; c < nch; ++c) {
                const uint32_t bb = sb + (c & 1) * LY::BUF;
                if (!mbar_wait(&bars.full[c & 1], (c >> 1) & 1, status)) { fail(); break; }
                if (!mbar_wait(&bars.t2_full, c & 1, status)) { fail(); break; }
                if (c >= 1 && !mbar_wait(&bars.y_ready, (c - 1) & 1, status)) { fail(); break; }
                fence_after_sync();
                // state-independent part of round 1, ahead of the state: U' = -[0; T2_hi] V - [0; T2_lo] V
                const uint64_t dV = (BV == 32) ? make_desc(bb + LY::B_V, 0, 512, 4)
                                               : make_desc(bb + LY::B_V, C * 128, 1024, 2);
                mma_steps<C / 16>(tb + LY::cU, idU, dZ1, dV, oK0, oVT, false);
                mma_steps<C / 16>(tb + LY::cU, idU, dZ2, dV, oK0, oVT, true);
                mma_commit(&bars.t2_empty);
                // state part: D1 = [Q; Wk] [S_hi | S_lo]
                if (!mbar_wait(&bars.s_ready, c & 1, status)) { fail(); break; }
                fence_after_sync();
                const uint64_t dQW = make_desc(bb + LY::B_KQW + C * 128, 16, 1024, 2);
                mma_steps<DK / 16>(tb + LY::cD1, idS, dQW, dS2, oKQW, oMN, false);
                mma_commit(&bars.d1_full);
                // round 2: the state update first (on the critical path), then the output
                if (!mbar_wait(&bars.y_ready, c & 1, status)) { fail(); break; }
                fence_after_sync();
                const uint64_t dKt = make_desc(bb + LY::B_KQW, LY::KQW_BLK, 1024, 2);
                mma_steps<C / 16>(tb + LY::cD4, idesc_bf16(DK, N2, 1, 1), dKt, dDY2, oMN, oMN, false);
                mma_commit(&bars.d4_full);
                if (!mbar_wait(&bars.mq_full, c & 1, status)) { fail(); break; }
                mma_steps<C / 16>(tb + LY::cD3, idesc_bf16(128, N2, 0, 1), dMH, dY2, oK0, oMN, false);
                mma_steps<C / 16>(tb + LY::cD3, idesc_bf16(128, BV, 0, 1), dML, dY2, oK0, oMN, true);
                mma_commit(&bars.d3_full);
                mma_commit(&bars.mq_empty);
                mma_commit(&bars.empty[c & 1]);
            }
        }
    } else {
        // ---------------- epilogue: warps 0-3 ----------------
        __nv_bfloat16 *o = (__nv_bfloat16 *)p.o;
        float *sGam = (float *)(sm + LY::GATES);
        float *sD = sGam + C;
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
        if (own_d) store_row_pair<BV>(sm + LY::S, LY::S_BLK, d_row, Sreg);
        fence_async_smem();
        named_sync(1, EPI_THREADS);
        if (tid == 0) mbar_arrive(&bars.s_ready);
        for (int c = 0; c < nch; ++c) {
            const int c0 = c * C, n = min(C, T - c0);
            const uint8_t *buf = sm + (c & 1) * LY::BUF;
            if (!mbar_wait(&bars.full[c & 1], (c >> 1) & 1, status)) { fail(); break; }
            const float *g = reinterpret_cast<const float *>(buf + LY::B_G);
            const float g_last = g[C - 1];
            if (tid < C) {
                sGam[tid] = __expf(g[tid]);
                sD[tid] = tid < n ? __expf(g_last - g[tid]) : 0.f;
            }
            named_sync(1, EPI_THREADS);
            if (tid == 0) mbar_arrive(&bars.empty[c & 1]);  // g has been read
            // Y = U - X_s (rows 64..127 of D1), QS (rows 0..63)
            if (!mbar_wait(&bars.d1_full, c & 1, status)) { fail(); break; }
            fence_after_sync();
            float qs[BV];
            ld_pair_sum<BV>(tb, warp, LY::cD1, qs);
            if (warp >= 2) {
                const int t = tid - 64;
                float y[BV];
                ld_row<BV>(tb, warp, LY::cU, y);  // -U
                const bool wr = !(p.flags & kNoWrite);
#pragma unroll
                for (int j = 0; j < BV; ++j) y[j] = -(qs[j] + (wr ? y[j] : 0.f));
                store_row_pair<BV>(sm + LY::Y, LY::Y_BLK, t, y);
                const float dd = sD[t];
#pragma unroll
                for (int j = 0; j < BV; ++j) y[j] *= dd;
                store_row_pair<BV>(sm + LY::DY, LY::Y_BLK, t, y);
            }
            fence_async_smem();
            fence_before_sync();
            named_sync(1, EPI_THREADS);
            if (tid == 0) mbar_arrive(&bars.y_ready);
            // state update S^T <- e^{g_n} S^T + K^T D Y
            if (!mbar_wait(&bars.d4_full, c & 1, status)) { fail(); break; }
            fence_after_sync();
            {
                float x[BV];
                ld_pair_sum<BV>(tb, warp, LY::cD4, x);
                const float gC = __expf(g_last);
                if (own_d) {
#pragma unroll
                    for (int j = 0; j < BV; ++j) Sreg[j] = fmaf(gC, Sreg[j], x[j]);
                    store_row_pair<BV>(sm + LY::S, LY::S_BLK, d_row, Sreg);
                }
            }
            fence_async_smem();
            fence_before_sync();
            named_sync(1, EPI_THREADS);
            if (tid == 0) mbar_arrive(&bars.s_ready);
            // output O = diag(e^g) QS + Mqk Y (overlaps the next chunk's first MMAs)
            if (!mbar_wait(&bars.d3_full, c & 1, status)) { fail(); break; }
            fence_after_sync();
            if (warp < 2) {
                float x[BV];
                ld_pair_sum<BV>(tb, warp, LY::cD3, x);
                const int t = tid;
                if (t < n && !(p.flags & kNoOutput)) {
                    const float gt = sGam[t];
                    __nv_bfloat16 *dst = o + (((size_t)b * T + c0 + t) * H + h) * dv + v0;
#pragma unroll
                    for (int c8 = 0; c8 < BV / 8; ++c8) {
                        float r[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) r[j] = fmaf(gt, qs[c8 * 8 + j], x[c8 * 8 + j]);
                        uint4 pk;
                        pk.x = pack_bf16(r[0], r[1]);
                        pk.y = pack_bf16(r[2], r[3]);
                        pk.z = pack_bf16(r[4], r[5]);
                        pk.w = pack_bf16(r[6], r[7]);
                        *reinterpret_cast<uint4 *>(dst + c8 * 8) = pk;
                    }
                }
            }
            fence_before_sync();
            named_sync(1, EPI_THREADS);  // D3 read before the next chunk's round 2 overwrites it
        }
        if (p.S_final && own_d && !failed()) {
#pragma unroll
            for (int j = 0; j < BV; ++j) p.S_final[(head * dv + v0 + j) * DK + d_row] = Sreg[j];
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, LY::TCOLS);
}

// Host: the driver's tensor-map encoder, fetched once through the runtime (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 4-D map over a bf16 activation [B, T, H, d]: dims {d, H, T, B}, box {box_d, 1, C, 1}.
bool act_map(CUtensorMap *m, const void *base, int B, int T, int H, int d, int box_d) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)T * H * d * 2};
    const cuuint32_t box[4] = {(cuuint32_t)box_d, 1, (cuuint32_t)C, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapSwizzle sw = box_d * 2 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DK, int BV>
bool gdn_maps(const ScanArgs &a, GdnMaps *maps) {
    return act_map(&maps->k, a.k, a.B, a.T, a.H, DK, 64) && act_map(&maps->q, a.q, a.B, a.T, a.H, DK, 64) &&
           act_map(&maps->v, a.v, a.B, a.T, a.H, a.dv, BV);
}

template <int DK, int BV>
cudaError_t launch_gdn_prep_t(const ScanArgs &a, void *ws, cudaStream_t s) {
    const int nch = (a.T + C - 1) / C;
    GdnMaps maps;
    if (!gdn_maps<DK, BV>(a, &maps)) return cudaErrorInvalidValue;
    using LY = PrepLayout<DK>;
    auto kern = gdn_prep_kernel<DK>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)LY::BYTES);
    if (err != cudaSuccess) return err;
    dim3 grid(nch, a.H, a.B);
    launch_probe_mark(s);
    kern<<<grid, NT, LY::BYTES, s>>>(a, maps, (uint8_t *)ws, nch);
    return cudaGetLastError();
}

template <int DK, int BV>
cudaError_t launch_gdn_state_t(const ScanArgs &a, const void *ws, cudaStream_t s) {
    const int nch = (a.T + C - 1) / C;
    GdnMaps maps;
    if (!gdn_maps<DK, BV>(a, &maps)) return cudaErrorInvalidValue;
    using LY = StateLayout<DK, BV>;
    static_assert(LY::BYTES <= 227 * 1024, "shared memory budget");
    auto kern = gdn_state_kernel<DK, BV>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)LY::BYTES);
    if (err != cudaSuccess) return err;
    dim3 grid(a.dv / BV, a.H, a.B);
    launch_probe_mark(s);
    kern<<<grid, ST_THREADS, LY::BYTES, s>>>(a, maps, (const uint8_t *)ws, nch);
    return cudaGetLastError();
}

}  // namespace

// Workspace bytes of the two-kernel GDN path: the status block plus one record per chunk.
size_t gdn_workspace_bytes(int B, int H, int T, int dk) {
    const size_t nch = (size_t)((T + C - 1) / C);
    const size_t rec = dk == 128 ? GdnRec<128>::BYTES : GdnRec<64>::BYTES;
    return kRecOffset + (size_t)B * H * nch * rec;
}

// The per-chunk records (prep) and the in-order pass over them (state); records depend only on
// q, k, alpha, beta, so several state passes over the same tokens can share one prep.
cudaError_t launch_gdn_prep(const ScanArgs &a, void *ws, cudaStream_t s) {
    if (a.T <= 0) return cudaSuccess;
    return a.dk == 128 ? launch_gdn_prep_t<128, 32>(a, ws, s) : launch_gdn_prep_t<64, 64>(a, ws, s);
}

cudaError_t launch_gdn_state(const ScanArgs &a, const void *ws, cudaStream_t s) {
    return a.dk == 128 ? launch_gdn_state_t<128, 32>(a, ws, s) : launch_gdn_state_t<64, 64>(a, ws, s);
}

cudaError_t launch_scan_gdn(const ScanArgs &a, void *ws, cudaStream_t s) {
    cudaError_t err = launch_gdn_prep(a, ws, s);
    if (err != cudaSuccess) return err;
    return launch_gdn_state(a, ws, s);
}

}  // namespace prism
