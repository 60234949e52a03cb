// scan_gdn.cu -- the chunked scan forward on the tcgen05 tensor cores as two kernels: a per-chunk
// prep that runs for every (batch, head, chunk) at once, and an in-order state kernel.
//
// The chunk form ("Sequential Parallel Duality in Prefix Scannable Models", method overview:
// chunk, encode, scan; exact because the per-token affine elements E_t = alpha_t (I - beta_t k_t
// k_t^T), f_t = sum_l u w^T compose associatively).  Per chunk of C = 64 tokens with entry state S,
// g_t = sum_{r<=t} log alpha_r, Gamma_{t,i} = e^{g_t - g_i}, D_i = e^{g_n - g_i}:
//   A = strict(diag(beta) Gamma o K K^T),  Mqk = incl(Gamma o Q K^T),  T = (I + A)^{-1},
//   Wk = T diag(beta e^g) K;
//   Gated-DeltaNet write (u = beta v, w = k):  U = T diag(beta) V;
//   rank-L write:  P_l = strict(diag(beta) Gamma o K W_l^T),  Mqw_l = incl(Gamma o Q W_l^T),
//     U = -X_u = -T sum_l P_l U_l,  O_w = sum_l Mqw_l U_l,  F_w = sum_l W_l^T D U_l;
//   Y = U - Wk S^T,   O = diag(e^g) Q S^T + Mqk Y (+ O_w),   S'^T = e^{g_n} S^T + K^T D Y (+ F_w),
// which is the token recurrence S_t = alpha_t S_{t-1}(I - beta_t k_t k_t^T) + sum_l u_{t,l}
// w_{t,l}^T, o_t = S_t q_t (PRISM, gist.science explainer, technical summary 2.1 and 2.2;
// banbantang.com PRISM article, section 1(4): the GDN forget and rank-1 write) unrolled over the
// chunk.  Everything but the last line depends only on the chunk's own tokens: the prep kernels
// (`gdn_prep_kernel`, `lrank_prep_kernel`) compute it for all chunks in parallel and write a
// per-chunk record to the workspace, laid out as the shared-memory images the state kernel reads;
// `gdn_state_kernel` then walks the chunks of one (batch, head, value slice) in order with the
// fp32 state on chip, prefetching the next chunk's tiles (TMA, double buffered).  Prep runs over
// chunks last-first, so the records the state kernel needs first are the ones most recently
// written and most likely still in L2.
//
// Operands that are rounded intermediate results (Mqk, T, Y, S and on the rank-L route P, Mqw,
// D U, sum P U) are kept as an unevaluated bf16 pair x = hi + lo (lo = bf16(x - hi)); a product is
// then a_hi b_hi + a_hi b_lo + a_lo b_hi, about 16 significant bits.  The inputs q, k, v, u, w are
// exact bf16.  A tcgen05.mma issued by one thread costs about 53 cycles whatever its N up to 128
// (measured on B200), so the kernels issue few, wide MMAs: hi and lo halves of an operand sit side
// by side along N, and two 64-row operands are stacked into one M = 128 instruction.  Every wait is
// a bounded mbarrier poll that records PRISM_ERR_TIMEOUT when it runs out.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "chunk_common.cuh"

namespace prism {
namespace {

constexpr int NT = 128;  // prep threads

// N consecutive TMEM columns of this thread's lane (N = 4, 8, 16 or 32; warp-collective).
template <int N>
__device__ __forceinline__ void tmem_ld_n(uint32_t a, float (&v)[N]) {
    if constexpr (N == 4) tmem_ld4(a, v);
    else if constexpr (N == 8) tmem_ld8(a, v);
    else if constexpr (N == 16) tmem_ld16(a, v);
    else tmem_ld32(a, v);
}

// N fp32 values at (row, col .. col+N-1) of K-major SW128 tiles as a bf16 hi / lo pair (N = 16, 32).
template <int N>
__device__ __forceinline__ void store_split_n(uint8_t *hi, uint8_t *lo, int row, int col, const float *x) {
    if constexpr (N == 32) {
        store32_split(hi, lo, row, col, x);
    } else {
#pragma unroll
        for (int c8 = 0; c8 < N / 8; ++c8) {
            uint4 h, l;
            split8(x + c8 * 8, h, l);
            const uint32_t off = sw128_off(row, col + c8 * 8, 0);
            st16(hi, off, h);
            st16(lo, off, l);
        }
    }
}

// Value-slice width of the state kernel for a key width: 4 slices of 32 at d = 128, one of 64 at
// d = 64 (the Gated-DeltaNet route has dv = dk).
template <int DK>
constexpr int kBV = DK == 128 ? 32 : 64;

// TMA descriptors of the bf16 activations, viewed as 4-D {d, H, T, B} (innermost first) so that
// a box {64, 1, 64, 1} is one head's chunk of 64 columns; rows past T read as zeros.
struct GdnMaps {
    CUtensorMap k, q, v;
};

// One workspace record per (b, h, chunk).  The rank-L record (RL) adds the write's own terms:
// O_w = sum_l Mqw_l U_l and F_w = sum_l W_l^T D U_l; its U slot holds -X_u = -T sum_l P_l U_l.
template <int DK, bool RL = false, int BV_ = kBV<DK>>
struct GdnRec {
    static constexpr int DV = DK, BV = BV_;
    static constexpr uint32_t WK_BLK = C * 128;                  // 64 rows x 128 B per 64 columns
    static constexpr uint32_t WK = 0;                             // Wk hi, bf16, K-major SW128
    static constexpr uint32_t WKL = WK + WK_BLK * (DK / 64);      // Wk lo (= bf16(Wk - hi)), same layout
    static constexpr uint32_t MQK = WKL + WK_BLK * (DK / 64);     // Mqk hi (rows 0..63), lo (64..127)
    static constexpr uint32_t U_SLICE = C * BV * 4;               // U, fp32, one value slice
    static constexpr uint32_t U = MQK + 2 * C * 128;
    static constexpr uint32_t G = U + U_SLICE * (DV / BV);        // g_t, 64 floats
    static constexpr uint32_t OW_SLICE = C * BV * 4;              // O_w, fp32, one value slice
    static constexpr uint32_t OW = G + 1024;                      // O_w slices [t][BV], XOR-swizzled (rank L)
    static constexpr uint32_t FW_SLICE = DK * BV * 4;             // F_w, fp32, one value slice
    static constexpr uint32_t FW = OW + (RL ? C * DV * 4 : 0);    // F_w slices [d][BV], XOR-swizzled
    static constexpr uint32_t BYTES = FW + (RL ? FW_SLICE * (DV / BV) : 0);
};
constexpr size_t kRecOffset = 1024;  // records start after the status block

// Byte offset of U[t][j] in one value slice of BV fp32 columns: 16-byte chunks XORed with t % 8
// (t % 4 for BV = 16, whose rows hold four chunks), so that consecutive rows read at one column
// hit different bank groups.
template <int BV>
__device__ __forceinline__ uint32_t u_off(int t, int j) {
    constexpr uint32_t mask = BV >= 32 ? 7u : (uint32_t)BV / 4 - 1;
    return (uint32_t)t * BV * 4 + ((((uint32_t)j >> 2) ^ ((uint32_t)t & mask)) << 4) + ((uint32_t)j & 3) * 4;
}

// ------------------------------------------------------------------------------------------------
// prep: one CTA per (chunk, head, batch)

// 55 KB at either width, so four CTAs share an SM.  At d = 128 the T pair tiles live in the Q
// rows (free once G is done); V replaces K once Wk is done; U is staged over all of it at the end.
template <int DK>
struct PrepLayout {
    static constexpr uint32_t KQ_BLK = 2 * C * 128;     // [K; Q] rows of one 64-column block
    static constexpr uint32_t KQ = 0;
    static constexpr uint32_t T1 = DK == 128 ? KQ + C * 128 : KQ + KQ_BLK;
    static constexpr uint32_t T1L = DK == 128 ? KQ + KQ_BLK + C * 128 : T1 + C * 128;
    static constexpr uint32_t AF = DK == 128 ? KQ + 2 * KQ_BLK : T1L + C * 128;  // fp32 A, solved in place into T
    static constexpr uint32_t TMP = AF + C * AS * 4;
    static constexpr uint32_t GATES = TMP + kSolveTmpFloats * 4;
    static constexpr uint32_t BYTES = GATES + 3 * C * 4 + 1024;
    static_assert(KQ_BLK * (DK / 64) >= (uint32_t)C * DK * 4, "U staging fits over K and V");
    static_assert(4 * (BYTES + 1024 + 64) <= 228 * 1024, "four CTAs share an SM");
};

// 8 warps, 4 CTAs per SM (64 registers a thread): warp w reads TMEM lane quarter w % 4, and warps
// w and w + 4 split the columns of every epilogue; the solve runs on warps 0-3.
constexpr int PREP_THREADS = 256;

template <int DK, int BV_>
__global__ void __launch_bounds__(PREP_THREADS, 4) gdn_prep_kernel(ScanArgs p, const __grid_constant__ GdnMaps maps,
                                                                  uint8_t *ws, int nch) {
    using LY = PrepLayout<DK>;
    using RC = GdnRec<DK, false, BV_>;
    constexpr int DV = RC::DV, BV = RC::BV;
    constexpr int NTH = PREP_THREADS, NH = NTH / 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t mma_bar, ld_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int failed_sh;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, hs = warp >> 2;  // TMEM lane quarter, column split
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
    // the give-up test: no tile load is issued and every wait runs out after a short limit
    const bool stall = (p.flags & kStallPrep) != 0;
    const uint32_t lim = stall ? kStallTestPolls : kWaitPolls;

    // The gates first: loads issued after the tile loads wait behind their data in the SM's
    // memory pipeline (measured ~4000 cycles on the rank-L prep), and the first epilogue needs both.
    float g_alpha = 1.f, g_beta = 0.f;
    if (tid < C && tid < n) {
        const size_t bth = ((size_t)b * T + c0 + tid) * H + h;
        g_alpha = p.alpha[bth];
        g_beta = p.beta[bth];
    }
    // K and Q boxes by TMA (rows past the end of the sequence arrive as zeros: identity tokens)
    if (tid == 0) {
        mbar_init(&mma_bar, 1);
        mbar_init(&ld_bar, 1);
        mbar_fence_init();
        failed_sh = 0;
        if (!stall) {
            mbar_expect_tx(&ld_bar, 2 * (DK / 64) * C * 128);
            for (int blk = 0; blk < DK / 64; ++blk) {
                tma_load_4d(sm + LY::KQ + blk * LY::KQ_BLK, &maps.k, blk * 64, h, c0, b, &ld_bar);
                tma_load_4d(sm + LY::KQ + blk * LY::KQ_BLK + C * 128, &maps.q, blk * 64, h, c0, b, &ld_bar);
            }
        }
    }
    if (warp == 0) tmem_alloc(&tmem_base_sh, 128);
    if (tid < C) {
        sG[tid] = tid < n ? logf(g_alpha) : 0.f;
        sBeta[tid] = g_beta;
    }
    __syncthreads();
    if (warp == 0) {
        const float x0 = warp_inclusive_scan(sG[lane], lane);
        const float x1 = warp_inclusive_scan(sG[32 + lane], lane) + __shfl_sync(0xffffffffu, x0, 31);
        sG[lane] = x0;
        sG[32 + lane] = x1;
    }
    if (!mbar_wait(&ld_bar, 0, p.status, lim)) failed_sh = 1;
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
    if (!mbar_wait(&mma_bar, 0, p.status, lim)) failed_sh = 1;
    fence_after_sync();
    __syncthreads();
    bool ok = failed_sh == 0;  // uniform across the CTA
    if (ok) {
        const int t = (q & 1) * 32 + lane;
        const float gt = sG[t], bt = sBeta[t];
        {
            const int cc = hs * 32;
            float gr[32];
            tmem_ld32(taddr(tb, 32 * q, cc), gr);
            tmem_wait_ld();
            if (q < 2) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int i = cc + j;
                    gr[j] = (i < t) ? bt * __expf(gt - sG[i]) * gr[j] : 0.f;
                }
                vst<32>(sA + t * AS + cc, gr);
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int i = cc + j;
                    gr[j] = (i <= t) ? __expf(gt - sG[i]) * gr[j] : 0.f;
                }
                store32_split(rec + RC::MQK, rec + RC::MQK + C * 128, t, cc, gr);
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    // T diag(beta scale) as a bf16 hi / lo pair into the T1 tiles (scale = e^g for Wk, 1 for U)
    auto store_t_pair = [&](bool with_gamma) {
        for (int e = tid; e < C * (C / 8); e += NTH) {
            const int t = e / (C / 8), c8 = e % (C / 8);
            float a[8];
            vld<8>(sA + t * AS + c8 * 8, a);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = c8 * 8 + j;
                a[j] = (i <= t) ? a[j] * sBeta[i] * (with_gamma ? sGam[i] : 1.f) : 0.f;
            }
            uint4 hv, lv;
            split8(a, hv, lv);
            const uint32_t off = sw128_off(t, c8 * 8, 0);
            st16(sm + LY::T1, off, hv);
            st16(sm + LY::T1L, off, lv);
        }
    };
    if (ok) {
        // on warps 0-3 (measured faster here than spreading it over all 8 warps)
        if (tid < 128) solve_unit_lower<128>(sA, sA, sTmp, tid, [] { named_sync(2, 128); });
        __syncthreads();
        store_t_pair(true);
    }
    sync_for_mma();
    // Wk = T diag(beta gamma) K  (M = 64, N = DK; K read as an MN-major operand)
    if (ok && tid == 0) {
        const uint32_t id = idesc_bf16(64, DK, 0, 1);
        const uint64_t dK = make_desc(sb + LY::KQ, LY::KQ_BLK, 1024, 2);
        mma_steps<C / 16>(tb, id, make_desc(sb + LY::T1, 16, 1024, 2), dK, ok0, omn, false);
        mma_steps<C / 16>(tb, id, make_desc(sb + LY::T1L, 16, 1024, 2), dK, ok0, omn, true);
        mma_commit(&mma_bar);
    }
    __syncwarp();
    if (ok && !mbar_wait(&mma_bar, 1, p.status, lim)) failed_sh = 1;
    fence_after_sync();
    __syncthreads();
    ok = failed_sh == 0;
    // V into the K rows, which no MMA reads any more; it lands during the Wk epilogue
    const bool v_issued = ok;
    if (ok && tid == 0) {
        mbar_expect_tx(&ld_bar, (DV / 64) * C * 128);
        for (int blk = 0; blk < DV / 64; ++blk)
            tma_load_4d(sm + LY::KQ + blk * LY::KQ_BLK, &maps.v, blk * 64, h, c0, b, &ld_bar);
    }
    // M = 64 accumulators: row r sits in lane 32 (r / 16) + r % 16
    const bool own_t = lane < 16;
    const int t_row = 16 * q + lane;
    if (ok) {
#pragma unroll
        for (int cc = hs * (DK / NH); cc < (hs + 1) * (DK / NH); cc += 32) {
            float x[32];
            tmem_ld32(taddr(tb, 32 * q, cc), x);
            tmem_wait_ld();
            if (own_t) store32_split(rec + RC::WK, rec + RC::WKL, t_row, cc, x, RC::WK_BLK);
        }
    }
    fence_before_sync();
    __syncthreads();
    // U = T diag(beta) V  (M = 64, N = DV; V read as an MN-major operand from the K rows)
    if (ok) store_t_pair(false);  // the Wk MMA has completed: the T1 tiles are free
    if (ok && !mbar_wait(&ld_bar, 1, p.status, lim)) failed_sh = 1;
    sync_for_mma();
    ok = failed_sh == 0;
    if (ok && tid == 0) {
        const uint32_t id = idesc_bf16(64, DV, 0, 1);
        const uint64_t dV = make_desc(sb + LY::KQ, LY::KQ_BLK, 1024, 2);
        mma_steps<C / 16>(tb, id, make_desc(sb + LY::T1, 16, 1024, 2), dV, ok0, omn, false);
        mma_steps<C / 16>(tb, id, make_desc(sb + LY::T1L, 16, 1024, 2), dV, ok0, omn, true);
        mma_commit(&mma_bar);
    }
    __syncwarp();
    if (ok && !mbar_wait(&mma_bar, 0, p.status, lim)) failed_sh = 1;
    fence_after_sync();
    __syncthreads();
    ok = failed_sh == 0;
    // U: TMEM -> the record's slice layout, staged over the K / Q rows (everything there was read
    // by completed MMAs), then one bulk store
    if (ok) {
        uint8_t *stage = sm + LY::KQ;
#pragma unroll
        for (int cc = hs * (DV / NH); cc < (hs + 1) * (DV / NH); cc += 32) {
            float x[32];
            tmem_ld32(taddr(tb, 32 * q, cc), x);
            tmem_wait_ld();
            if (own_t) {
#pragma unroll
                for (int j4 = 0; j4 < 32; j4 += 4) {
                    const int j = cc + j4;
                    *reinterpret_cast<float4 *>(stage + (j / BV) * RC::U_SLICE + u_off<BV>(t_row, j % BV)) =
                        make_float4(x[j4], x[j4 + 1], x[j4 + 2], x[j4 + 3]);
                }
            }
        }
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    if (ok && tid == 0) {
        bulk_s2g(rec + RC::U, sm + LY::KQ, (uint32_t)(C * DV * 4));
        bulk_commit();
        bulk_wait_read();  // the staging buffer is read out before the CTA frees it; the kernel's
                           // end makes the writes visible to the next launch
    }
    // after a failure, let the tile loads still in flight land before the CTA exits
    if (!ok && tid == 0 && !stall) mbar_wait(&ld_bar, v_issued ? 1 : 0, nullptr);
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 128);
}

// ------------------------------------------------------------------------------------------------
// rank-L prep: one CTA per (chunk, head, batch), all value columns at once
//
// The state-independent part of a chunk with the write sum_l u_l w_l^T:
//   G = [K; Q] K^T -> A, Mqk;  T = (I + A)^{-1};  Wk = T diag(beta e^g) K;
//   per l:  G_l = [K; Q] W_l^T -> P_l = strict(diag(beta) Gamma o K W_l^T), Mqw_l = incl(Gamma o Q W_l^T),
//           sum P_l U_l,  O_w += Mqw_l U_l,  F_w += W_l^T D U_l;
//   X_u = T sum_l P_l U_l.
// The record gets Wk, Mqk, -X_u (in the U slot, so that the state kernel's Y = U - Wk S^T holds for
// both writes), O_w, F_w and g.

struct LMaps {
    CUtensorMap k, q, w, u;  // w, u viewed as {d, H*L, T, B}: box row (h, l) = h L + l
};

template <int DK>
struct LPrepLayout {
    static constexpr uint32_t KQ_BLK = 2 * C * 128;     // [K; Q] rows of one 64-column block
    static constexpr uint32_t BLK = C * 128;            // one 64-column block of a C-row tile
    // W_l buffers: two (the next rank's W loads while this one's is read); U_l buffers: two at
    // d = 128, one at d = 64, where shared memory is kept small enough for two CTAs per SM
    static constexpr int NBU = DK == 128 ? 2 : 1;
    static constexpr uint32_t TILE = BLK * (DK / 64);   // one C x DK bf16 tile
    static constexpr uint32_t KQ = 0;
    static constexpr uint32_t W = KQ + KQ_BLK * (DK / 64);   // W_l, K-major (rows t)
    static constexpr uint32_t U = W + 2 * TILE;              // U_l, [t][dv] (MN-major B operand)
    static constexpr uint32_t DU = U + NBU * TILE;           // D U_l hi, lo; later sum P U hi, lo
    static constexpr uint32_t DUL = DU + BLK * (DK / 64);
    static constexpr uint32_t T1 = DUL + BLK * (DK / 64);    // T diag(beta gamma), then T: hi, lo
    static constexpr uint32_t T1L = T1 + BLK;
    // At d = 128 the solve (warps 0-7) and the rank loop (warps 8-15) run at the same time; at
    // d = 64 (8 warps, two CTAs per SM) one after the other.
    static constexpr bool SPLIT = DK == 128;
    // [P_l; Mqw_l] as two M = 128 operands: the lo rows after the T tiles, the hi rows after them
    // (SPLIT) or over the solve buffer (free once both T tiles are built)
    static constexpr uint32_t PL = T1L + BLK;
    static constexpr uint32_t MQWL = PL + BLK;
    static constexpr uint32_t AF = MQWL + BLK + (SPLIT ? 2 * BLK : 0);  // fp32 A, solved in place into T
    static constexpr uint32_t P = SPLIT ? MQWL + BLK : AF;
    static constexpr uint32_t MQW = P + BLK;
    // Mqk (hi, lo) staged for its bulk store: over the T tiles (SPLIT: the rank loop writes the
    // [P; Mqw] tiles while the solve runs) or over the lo [P; Mqw] tiles
    static constexpr uint32_t MQK_HI = SPLIT ? T1 : PL;
    static_assert(T1L == T1 + BLK && MQWL == PL + BLK && BLK == C * 128, "Mqk hi / lo staged adjacent");
    static constexpr uint32_t TMP = AF + C * AS * 4;
    static constexpr uint32_t GATES = TMP + kSolveTmpFloats * 4;   // g, beta, gamma, D
    // (SPLIT) the chunk's decay matrix e^{g_t - g_i} (i <= t, else 0), fp32 [C][AS] (rows padded
    // like A's, so that a warp reading 32 rows at one column spreads over the banks): every G
    // epilogue scales by it instead of recomputing its exponentials per thread
    static constexpr uint32_t DECAY = GATES + 4 * C * 4;
    static constexpr uint32_t BYTES = DECAY + (SPLIT ? C * AS * 4 : 0) + 1024;
    static_assert(KQ_BLK * (DK / 64) >= (uint32_t)C * DK * 4, "-X_u staging fits over K and Q");
    static_assert(SPLIT || MQW + BLK <= TMP, "the hi P / Mqw rows fit over the solve matrix");
    static_assert(!SPLIT || (MQW + BLK == AF && MQWL + BLK == P && (uint32_t)C * DK * 4 <= 4 * BLK),
                  "O_w is staged over the four [P; Mqw] tiles");
    static_assert(DK == 128 || 2 * (BYTES + 1024 + 64) <= 228 * 1024, "two CTAs share an SM at d = 64");
    // TMEM: G (64 columns, M = 128); Wk, then [sum P U; O_w] (M = 128), then X_u (DK columns);
    // F_w as its D U_hi and D U_lo halves (2 DK columns)
    static constexpr uint32_t cG = 0, cA = 64, cF = cA + DK;
    static constexpr uint32_t TCOLS = cF + 2 * DK <= 256 ? 256 : 512;
};

// One CTA per SM at d = 128 (its TMEM accumulators take 448 columns), with 16 warps; two CTAs per
// SM at d = 64 (256 columns and 112 KB of shared memory each), with 8 warps.  Warp w reads TMEM lane
// quarter w % 4; the warps sharing a quarter split the columns of every epilogue.
template <int DK>
constexpr int kLPrepThreads = DK == 128 ? 512 : 256;

template <int DK, int BV_>
__global__ void __launch_bounds__(kLPrepThreads<DK>, DK == 64 ? 2 : 1) lrank_prep_kernel(ScanArgs p, const __grid_constant__ LMaps maps,
                                                                      uint8_t *ws, int nch) {
    using LY = LPrepLayout<DK>;
    constexpr int NTH = kLPrepThreads<DK>;
    constexpr int NH = NTH / 128;  // column splits of an epilogue
    constexpr int CW = C / NH;     // columns of G a thread owns
    static_assert(CW == 32 || CW == 16, "the G epilogues move 16 or 32 columns a thread");
    using RC = GdnRec<DK, true, BV_>;
    constexpr int DV = RC::DV, BV = RC::BV;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t mma_bar, ld_bar, w_bar[2], u_bar[2];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int failed_sh;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, hs = warp >> 2;  // TMEM lane quarter, column split
    const int c = nch - 1 - blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int H = p.H, T = p.T, L = p.L;
    constexpr int NBU = LY::NBU;
    const int c0 = c * C, n = min(C, T - c0);
    uint8_t *rec = ws + kRecOffset + (((size_t)b * H + h) * nch + c) * RC::BYTES;
    float *sA = (float *)(sm + LY::AF);
    float *sTmp = (float *)(sm + LY::TMP);
    float *sG = (float *)(sm + LY::GATES);
    float *sBeta = sG + C;
    float *sGam = sBeta + C;
    float *sD = sGam + C;
    const uint32_t sb = smem_u32(sm);
    // the give-up test: no tile load is issued and every wait runs out after a short limit
    const bool stall = (p.flags & kStallPrep) != 0;
    const uint32_t lim = stall ? kStallTestPolls : kWaitPolls;
    uint32_t mph = 0, lph = 0;  // phases of mma_bar and ld_bar
    // W_l into W buffer l % 2 (completing on w_bar[l % 2]), U_l into U buffer l % NBU (u_bar)
    auto load_w = [&](int l) {
        const int bi = l & 1;
        mbar_expect_tx(&w_bar[bi], LY::TILE);
        for (int blk = 0; blk < DK / 64; ++blk)
            tma_load_4d(sm + LY::W + bi * LY::TILE + blk * LY::BLK, &maps.w, blk * 64, h * L + l, c0, b, &w_bar[bi]);
    };
    auto load_u = [&](int l) {
        const int bi = l % NBU;
        mbar_expect_tx(&u_bar[bi], LY::TILE);
        for (int blk = 0; blk < DK / 64; ++blk)
            tma_load_4d(sm + LY::U + bi * LY::TILE + blk * LY::BLK, &maps.u, blk * 64, h * L + l, c0, b, &u_bar[bi]);
    };
    int w_issued = 0, u_issued = 0;  // ranks whose W / U loads were issued (thread 0)

    // The gates first: loads issued after the tile loads wait behind their data in the SM's
    // memory pipeline (measured ~4000 cycles), and the first epilogue needs both.
    float g_alpha = 1.f, g_beta = 0.f;
    if (tid < C && tid < n) {
        const size_t bth = ((size_t)b * T + c0 + tid) * H + h;
        g_alpha = p.alpha[bth];
        g_beta = p.beta[bth];
    }
    if (tid == 0) {
        mbar_init(&mma_bar, 1);
        mbar_init(&ld_bar, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&w_bar[i], 1);
            mbar_init(&u_bar[i], 1);
        }
        mbar_fence_init();
        failed_sh = 0;
        if (!stall) {
            mbar_expect_tx(&ld_bar, 2 * (DK / 64) * C * 128);
            for (int blk = 0; blk < DK / 64; ++blk) {
                tma_load_4d(sm + LY::KQ + blk * LY::KQ_BLK, &maps.k, blk * 64, h, c0, b, &ld_bar);
                tma_load_4d(sm + LY::KQ + blk * LY::KQ_BLK + C * 128, &maps.q, blk * 64, h, c0, b, &ld_bar);
            }
            // the first ranks' W_l, U_l load while A, T and Wk are computed
            for (; w_issued < L && w_issued < 2; ++w_issued) load_w(w_issued);
            for (; u_issued < L && u_issued < NBU; ++u_issued) load_u(u_issued);
        }
    }
    if (warp == 0) tmem_alloc(&tmem_base_sh, LY::TCOLS);
    if (tid < C) {
        sG[tid] = tid < n ? logf(g_alpha) : 0.f;
        sBeta[tid] = g_beta;
    }
    __syncthreads();
    if (warp == 0) {
        const float x0 = warp_inclusive_scan(sG[lane], lane);
        const float x1 = warp_inclusive_scan(sG[32 + lane], lane) + __shfl_sync(0xffffffffu, x0, 31);
        sG[lane] = x0;
        sG[32 + lane] = x1;
    }
    if (!mbar_wait(&ld_bar, lph++ & 1, p.status, lim)) failed_sh = 1;
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tb = tmem_base_sh;
    if (tid < C) {
        sGam[tid] = expf(sG[tid]);
        sD[tid] = tid < n ? expf(sG[C - 1] - sG[tid]) : 0.f;
        reinterpret_cast<float *>(rec + RC::G)[tid] = sG[tid];
    }
    // thread 0 issued MMAs: commit, and every thread waits (bounded) for their completion
    auto mma_done = [&](bool issued) -> bool {
        if (tid == 0 && issued) mma_commit(&mma_bar);
        __syncwarp();
        if (issued && !mbar_wait(&mma_bar, mph & 1, p.status, lim)) failed_sh = 1;
        if (issued) mph++;
        fence_after_sync();
        __syncthreads();
        return failed_sh == 0;
    };
    // the same wait, for MMAs whose commit thread 0 already issued
    auto mma_done_committed = [&](bool issued) -> bool {
        __syncwarp();
        if (issued && !mbar_wait(&mma_bar, mph & 1, p.status, lim)) failed_sh = 1;
        if (issued) mph++;
        fence_after_sync();
        __syncthreads();
        return failed_sh == 0;
    };
    auto okq = [](int ks) { return (uint64_t)koff_k_sw128(ks, LY::KQ_BLK); };
    auto okb = [](int ks) { return (uint64_t)koff_k_sw128(ks, LY::BLK); };
    auto ok0 = [](int ks) { return (uint64_t)koff_k_sw128(ks, 0); };
    auto omn = [](int ks) { return (uint64_t)koff_mn_sw128(ks); };
    const uint64_t dKQ = make_desc(sb + LY::KQ, 16, 1024, 2);

    // G = [K; Q] K^T  ->  A (fp32, shared) and Mqk (hi / lo, straight to the record)
    bool ok = failed_sh == 0;
    if (ok && tid == 0) {
        mma_steps<DK / 16>(tb + LY::cG, idesc_bf16(128, C, 0, 0), dKQ, dKQ, okq, okq, false);
        mma_commit(&mma_bar);
    }
    // Every G epilogue (this one and one per rank) gives this thread row t_g, columns cg ..
    // cg + 31, and scales them by the same factors, computed once while the MMA runs:
    // beta_t e^{g_t - g_i} for i < t on the K rows (lane quarters 0-1: A and P_l), e^{g_t - g_i}
    // for i <= t on the Q rows (quarters 2-3: Mqk and Mqw_l).
    const int t_g = (q & 1) * 32 + lane, cg = hs * CW;
    float *sE = (float *)(sm + LY::DECAY);
    // the factors of a G epilogue row t_g, columns c0 .. c0 + N: from the decay matrix (SPLIT) or
    // computed here
    auto g_factors = [&](int c0, auto &f) {
        constexpr int N = sizeof(f) / sizeof(float);
        const float sc = q < 2 ? sBeta[t_g] : 1.f;
        if constexpr (LY::SPLIT) {
            vld<N>(sE + t_g * AS + c0, f);
#pragma unroll
            for (int j = 0; j < N; ++j) f[j] = (q < 2 && c0 + j == t_g) ? 0.f : sc * f[j];
        } else {
            const float gt = sG[t_g];
#pragma unroll
            for (int j = 0; j < N; ++j) {
                const int i = c0 + j;
                f[j] = (q < 2 ? i < t_g : i <= t_g) ? sc * __expf(gt - sG[i]) : 0.f;
            }
        }
    };
    if constexpr (LY::SPLIT) {  // the decay matrix while the MMA runs: 8 exponentials a thread
        for (int e = tid; e < C * C; e += NTH) {
            const int t = e / C, i = e % C;
            sE[t * AS + i] = i <= t ? __expf(sG[t] - sG[i]) : 0.f;
        }
    }
    float dec[CW];
    if constexpr (LY::SPLIT) {
        __syncthreads();  // the decay matrix is complete
    }
    g_factors(cg, dec);
    ok = mma_done_committed(ok);
    // the record is written by bulk stores from shared memory that is idle at that point (Mqk over
    // the lo [P; Mqw] tiles, the Wk pair over the D U tiles, O_w over K / Q, F_w over W / U):
    // whole contiguous pieces instead of 16-byte stores to 64 different rows per warp
    if (ok) {
        float gr[CW];
        tmem_ld_n<CW>(taddr(tb, 32 * q, LY::cG + cg), gr);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < CW; ++j) gr[j] *= dec[j];
        if (q < 2) vst<CW>(sA + t_g * AS + cg, gr);
        else store_split_n<CW>(sm + LY::MQK_HI, sm + LY::MQK_HI + C * 128, t_g, cg, gr);
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    // Mqk hi then lo (two adjacent tiles, as in the record), stored by thread 0, which waits for
    // the store to have read them before those tiles are written again (by the T pair at d = 128,
    // by the first P / Mqw epilogue at d = 64)
    constexpr int kRankIssuer = LY::SPLIT ? 256 : 0;
    constexpr int kSolveThreads = 256;  // (SPLIT) the solve's warps: 0-7
    if (ok && tid == 0) {
        bulk_s2g(rec + RC::MQK, sm + LY::MQK_HI, 2 * C * 128);
        bulk_commit();
    }
    // T pair tiles: T diag(beta gamma) for Wk, then T itself for X_u
    auto store_t_pair = [&](bool scaled, int first, int step) {
        for (int e = first; e < C * (C / 8); e += step) {
            const int t = e / (C / 8), c8 = e % (C / 8);
            float a[8];
            vld<8>(sA + t * AS + c8 * 8, a);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = c8 * 8 + j;
                a[j] = (i <= t) ? (scaled ? a[j] * sBeta[i] * sGam[i] : a[j]) : 0.f;
            }
            uint4 hv, lv;
            split8(a, hv, lv);
            const uint32_t off = sw128_off(t, c8 * 8, 0);
            st16(sm + LY::T1, off, hv);
            st16(sm + LY::T1L, off, lv);
        }
    };
    if constexpr (!LY::SPLIT) {
        if (ok) {
            solve_unit_lower<NTH>(sA, sA, sTmp, tid);  // ends with a CTA barrier
            store_t_pair(true, tid, NTH);
        }
        sync_for_mma();
        // Wk = T diag(beta gamma) K  (M = 64; row r of an M = 64 accumulator sits in lane 32 (r / 16) + r % 16)
        const uint64_t dKmn = make_desc(sb + LY::KQ, LY::KQ_BLK, 1024, 2);
        if (ok && tid == 0) {
            const uint32_t id = idesc_bf16(64, DK, 0, 1);
            mma_steps<C / 16>(tb + LY::cA, id, make_desc(sb + LY::T1, 16, 1024, 2), dKmn, ok0, omn, false);
            mma_steps<C / 16>(tb + LY::cA, id, make_desc(sb + LY::T1L, 16, 1024, 2), dKmn, ok0, omn, true);
        }
        ok = mma_done(ok);
        const bool own_t = lane < 16;
        const int t_row = 16 * q + lane;
        if (ok) {
    #pragma unroll
            for (int cc = hs * (DK / NH); cc < (hs + 1) * (DK / NH); cc += 32) {
                float x[32];
                tmem_ld32(taddr(tb, 32 * q, LY::cA + cc), x);
                tmem_wait_ld();
                if (own_t) store32_split(sm + LY::DU, sm + LY::DUL, t_row, cc, x, LY::BLK);
            }
        }
        fence_async_smem();
        fence_before_sync();
        __syncthreads();
        if (ok && tid == 0) {  // Wk hi then lo: DU and DUL are adjacent, as WK and WKL in the record
            static_assert(LY::DUL == LY::DU + RC::WK_BLK * (DK / 64) && RC::WKL == RC::WK + RC::WK_BLK * (DK / 64) &&
                              LY::BLK == RC::WK_BLK,
                          "the staged Wk pair has the record's layout");
            bulk_s2g(rec + RC::WK, sm + LY::DU, 2 * RC::WK_BLK * (DK / 64));
            bulk_commit();
        }
        if (ok) store_t_pair(false, tid, NTH);  // the Wk MMA has completed: the T tiles are free

        // the write terms, one rank at a time.  G_l = [K; Q] W_l^T is issued together with the
        // previous rank's MMAs (W is double-buffered), so each rank waits for one MMA batch.
        const uint32_t idV = idesc_bf16(64, DV, 0, 1);
        auto issue_g = [&](int l) {  // thread 0, once W_l has landed
            const uint64_t dW = make_desc(sb + LY::W + (l & 1) * LY::TILE, 16, 1024, 2);
            mma_steps<DK / 16>(tb + LY::cG, idesc_bf16(128, C, 0, 0), dKQ, dW, okq, okb, false);
        };
        if (ok && tid == 0) {
            if (mbar_wait(&w_bar[0], 0, p.status, lim)) issue_g(0);
            else failed_sh = 1;
            bulk_wait_read();  // the staged Mqk and Wk are read out: the rank loop writes those tiles
        }
        ok = mma_done(ok);
        for (int l = 0; l < L && ok; ++l) {
            const uint32_t wb = LY::W + (l & 1) * LY::TILE, ub = LY::U + (l % NBU) * LY::TILE;
            const uint64_t dWmn = make_desc(sb + wb, LY::BLK, 1024, 2);
            const uint64_t dU = make_desc(sb + ub, LY::BLK, 1024, 2);
            if (tid == 0 && l + 2 < L) {  // the rank after the ones in flight: start it toward L2
                for (int blk = 0; blk < DK / 64; ++blk) {
                    tma_prefetch_4d(&maps.w, blk * 64, h * L + l + 2, c0, b);
                    tma_prefetch_4d(&maps.u, blk * 64, h * L + l + 2, c0, b);
                }
            }
            {   // P_l (rows of K W^T, quarters 0-1) and Mqw_l (rows of Q W^T, quarters 2-3) as pairs
                float gr[CW];
                tmem_ld_n<CW>(taddr(tb, 32 * q, LY::cG + cg), gr);
                tmem_wait_ld();
    #pragma unroll
                for (int j = 0; j < CW; ++j) gr[j] *= dec[j];
                store_split_n<CW>(sm + (q < 2 ? LY::P : LY::MQW), sm + (q < 2 ? LY::PL : LY::MQWL), t_g, cg, gr);
            }
            if (!mbar_wait(&u_bar[l % NBU], (l / NBU) & 1, p.status, lim)) failed_sh = 1;
            for (int e = tid; e < C * (DV / 8); e += NTH) {  // D U_l as a hi / lo pair
                const int t = e / (DV / 8), c8 = e % (DV / 8);
                const uint32_t off = sw128_off(t, c8 * 8, LY::BLK);
                const uint4 uv = *reinterpret_cast<const uint4 *>(sm + ub + off);
                const __nv_bfloat16 *hv = reinterpret_cast<const __nv_bfloat16 *>(&uv);
                float du[8];
    #pragma unroll
                for (int j = 0; j < 8; ++j) du[j] = sD[t] * __bfloat162float(hv[j]);
                uint4 dh, dl;
                split8(du, dh, dl);
                st16(sm + LY::DU, off, dh);
                st16(sm + LY::DUL, off, dl);
            }
            sync_for_mma();
            ok = failed_sh == 0;
            if (ok && tid == 0) {
                const bool acc = l > 0;
                // [sum P U; O_w] += [P_l; Mqw_l] U_l  (M = 128, accumulated over l in the Wk columns)
                const uint32_t idPU = idesc_bf16(128, DV, 0, 1);
                mma_steps<C / 16>(tb + LY::cA, idPU, make_desc(sb + LY::P, 16, 1024, 2), dU, ok0, omn, acc);
                mma_steps<C / 16>(tb + LY::cA, idPU, make_desc(sb + LY::PL, 16, 1024, 2), dU, ok0, omn, true);
                // F_w += W_l^T [D U_l hi | D U_l lo]  (M = DK: W_l read as an MN-major A operand;
                // N = 2 DV: the D U tiles sit side by side as one operand)
                const uint32_t idF = idesc_bf16(DK, 2 * DV, 1, 1);
                mma_steps<C / 16>(tb + LY::cF, idF, dWmn, make_desc(sb + LY::DU, LY::BLK, 1024, 2), omn, omn, acc);
                // the next rank's G (its epilogue read of the G columns above is complete)
                if (l + 1 < L) {
                    if (mbar_wait(&w_bar[(l + 1) & 1], ((l + 1) >> 1) & 1, p.status, lim)) issue_g(l + 1);
                    else failed_sh = 1;
                }
            }
            ok = mma_done(ok);
            // rank l's W and U buffers are free: W_{l+2} and U_{l+NBU} load into them
            if (ok && tid == 0) {
                if (w_issued < L) load_w(w_issued++);
                if (u_issued < L) load_u(u_issued++);
            }
        }
        // [sum P U; O_w]: the sum P U rows (lane quarters 0-1) become a hi / lo pair over the D U
        // tiles, the O_w rows (quarters 2-3) are staged over K / Q in the record's layout
        if (ok) {
            const int t = 32 * (q & 1) + lane;
    #pragma unroll
            for (int cc = hs * (DV / NH); cc < (hs + 1) * (DV / NH); cc += 32) {
                float x[32];
                tmem_ld32(taddr(tb, 32 * q, LY::cA + cc), x);
                tmem_wait_ld();
                if (q < 2) {
    #pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {
                        uint4 hv, lv;
                        split8(x + 8 * c8, hv, lv);
                        const uint32_t off = sw128_off(t, cc + 8 * c8, LY::BLK);
                        st16(sm + LY::DU, off, hv);
                        st16(sm + LY::DUL, off, lv);
                    }
                } else {  // in the record's value-slice layout
                    uint8_t *stage = sm + LY::KQ;
    #pragma unroll
                    for (int j4 = 0; j4 < 32; j4 += 4) {
                        const int j = cc + j4;
                        *reinterpret_cast<float4 *>(stage + (j / BV) * RC::OW_SLICE + u_off<BV>(t, j % BV)) =
                            make_float4(x[j4], x[j4 + 1], x[j4 + 2], x[j4 + 3]);
                    }
                }
            }
        }
        sync_for_mma();
        static_assert(C * DV * 4 <= LY::KQ_BLK * (DK / 64), "O_w fits over K and Q");
        static_assert(RC::FW_SLICE * (DV / BV) <= LY::DU - LY::W, "F_w fits over W and U");
        if (ok && tid == 0) {
            bulk_s2g(rec + RC::OW, sm + LY::KQ, C * DV * 4);
            bulk_commit();
        }
        // X_u = T (sum P U)  (M = 64, into the same columns)
        if (ok && tid == 0) {
            const uint64_t dPU = make_desc(sb + LY::DU, LY::BLK, 1024, 2);
            const uint64_t dPUL = make_desc(sb + LY::DUL, LY::BLK, 1024, 2);
            const uint64_t dT = make_desc(sb + LY::T1, 16, 1024, 2), dTL = make_desc(sb + LY::T1L, 16, 1024, 2);
            mma_steps<C / 16>(tb + LY::cA, idV, dT, dPU, ok0, omn, false);
            mma_steps<C / 16>(tb + LY::cA, idV, dT, dPUL, ok0, omn, true);
            mma_steps<C / 16>(tb + LY::cA, idV, dTL, dPU, ok0, omn, true);
            mma_commit(&mma_bar);
        }
        // F_w (its MMAs are complete) while X_u runs: the D U_hi and D U_lo halves summed; rows d:
        // lane = d for M = 128 (DK = 128), lanes 32q + r, r < 16, for M = 64
        if (ok) {
            const bool own_d = (DK == 128) ? true : (lane < 16);
            const int d_row = (DK == 128) ? 32 * q + lane : (16 * q + lane);
    #pragma unroll
            for (int cc = hs * (DV / NH); cc < (hs + 1) * (DV / NH); cc += 16) {
                float xh[16], xl[16];
                tmem_ld16(taddr(tb, 32 * q, LY::cF + cc), xh);
                tmem_ld16(taddr(tb, 32 * q, LY::cF + DV + cc), xl);
                tmem_wait_ld();
                if (own_d) {  // staged over W / U in the record's layout
    #pragma unroll
                    for (int j4 = 0; j4 < 16; j4 += 4) {
                        const int j = cc + j4;
                        *reinterpret_cast<float4 *>(sm + LY::W + (j / BV) * RC::FW_SLICE + u_off<BV>(d_row, j % BV)) =
                            make_float4(xh[j4] + xl[j4], xh[j4 + 1] + xl[j4 + 1], xh[j4 + 2] + xl[j4 + 2],
                                        xh[j4 + 3] + xl[j4 + 3]);
                    }
                }
            }
        }
        fence_async_smem();
        fence_before_sync();
        __syncthreads();
        if (ok && tid == 0) {
            bulk_s2g(rec + RC::FW, sm + LY::W, RC::FW_SLICE * (DV / BV));
            bulk_commit();
            bulk_wait_read_n<1>();  // the O_w store has read K / Q, where -X_u is staged next
        }
        ok = mma_done_committed(ok);
        // -X_u -> the U slot (staged over K and Q in the record's slice layout, one bulk store)
        if (ok) {
            uint8_t *stage = sm + LY::KQ;
    #pragma unroll
            for (int cc = hs * (DV / NH); cc < (hs + 1) * (DV / NH); cc += 32) {
                float x[32];
                tmem_ld32(taddr(tb, 32 * q, LY::cA + cc), x);
                tmem_wait_ld();
                if (own_t) {
    #pragma unroll
                    for (int j4 = 0; j4 < 32; j4 += 4) {
                        const int j = cc + j4;
                        *reinterpret_cast<float4 *>(stage + (j / BV) * RC::U_SLICE + u_off<BV>(t_row, j % BV)) =
                            make_float4(-x[j4], -x[j4 + 1], -x[j4 + 2], -x[j4 + 3]);
                    }
                }
            }
        }
        fence_async_smem();
        fence_before_sync();
        __syncthreads();
        if (ok && tid == 0) {
            bulk_s2g(rec + RC::U, sm + LY::KQ, (uint32_t)(C * DV * 4));
            bulk_commit();
            bulk_wait_read();  // the staging buffer is read out before the CTA frees it; the kernel's
                               // end makes the writes visible to the next launch
        }
    } else {
        // ---- d = 128: the solve (warps 0-7) and the rank loop (warps 8-15) at the same time; the
        // rank loop needs none of T (only Wk and X_u do, and they follow the join) ----
        constexpr int GS = kSolveThreads, RB = 256, GR = NTH - RB;  // the solve's and the rank loop's threads
        const bool r_issuer = tid == kRankIssuer;
        const uint32_t idV = idesc_bf16(64, DV, 0, 1);
        const uint64_t dKmn = make_desc(sb + LY::KQ, LY::KQ_BLK, 1024, 2);
        const bool own_t = lane < 16;
        const int t_row = 16 * q + lane;
        int w_next = stall ? 0 : (L < 2 ? L : 2), u_next = stall ? 0 : (L < NBU ? L : NBU);  // (issuer)
        if (tid < GS) {
            if (ok) {
                solve_unit_lower<GS>(sA, sA, sTmp, tid, [] { named_sync(3, GS); });
                if (tid == 0) bulk_wait_read();  // the Mqk staged over the T tiles is read out
                named_sync(3, GS);
                store_t_pair(true, tid, GS);  // T diag(beta gamma) for Wk
            }
        } else if (tid >= RB) {
            // The write terms, one rank at a time, on this group's 8 warps (TMEM lane quarter
            // warp % 4, two column halves).  G_l = [K; Q] W_l^T is issued together with the
            // previous rank's MMAs (W is double-buffered), so each rank waits for one MMA batch.
            constexpr int CWR = C / 2;
            const int cgr = ((warp - RB / 32) >> 2) * CWR;
            const int rt = tid - RB;
            float decr[CWR];  // the G epilogue factors of this thread's row and columns
            g_factors(cgr, decr);
            uint32_t rph = mph;  // mma_bar phases this group has waited for
            auto r_done = [&](bool issued) -> bool {  // the issuer commits; the group waits
                if (r_issuer && issued) mma_commit(&mma_bar);
                __syncwarp();
                if (issued && !mbar_wait(&mma_bar, rph & 1, p.status, lim)) failed_sh = 1;
                if (issued) rph++;
                fence_after_sync();
                named_sync(4, GR);
                return failed_sh == 0;
            };
            auto issue_g = [&](int l) {  // the issuer, once W_l has landed
                const uint64_t dW = make_desc(sb + LY::W + (l & 1) * LY::TILE, 16, 1024, 2);
                mma_steps<DK / 16>(tb + LY::cG, idesc_bf16(128, C, 0, 0), dKQ, dW, okq, okb, false);
            };
            bool rok = ok;
            if (rok && r_issuer) {
                if (mbar_wait(&w_bar[0], 0, p.status, lim)) issue_g(0);
                else failed_sh = 1;
            }
            rok = r_done(rok);
            for (int l = 0; l < L && rok; ++l) {
                const uint32_t wb = LY::W + (l & 1) * LY::TILE, ub = LY::U + (l % NBU) * LY::TILE;
                const uint64_t dWmn = make_desc(sb + wb, LY::BLK, 1024, 2);
                const uint64_t dU = make_desc(sb + ub, LY::BLK, 1024, 2);
                if (r_issuer && l + 2 < L) {  // the rank after the ones in flight: start it toward L2
                    for (int blk = 0; blk < DK / 64; ++blk) {
                        tma_prefetch_4d(&maps.w, blk * 64, h * L + l + 2, c0, b);
                        tma_prefetch_4d(&maps.u, blk * 64, h * L + l + 2, c0, b);
                    }
                }
                {   // P_l (rows of K W^T, quarters 0-1) and Mqw_l (rows of Q W^T, quarters 2-3) as pairs
                    float gr[CWR];
                    tmem_ld_n<CWR>(taddr(tb, 32 * q, LY::cG + cgr), gr);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < CWR; ++j) gr[j] *= decr[j];
                    store_split_n<CWR>(sm + (q < 2 ? LY::P : LY::MQW), sm + (q < 2 ? LY::PL : LY::MQWL), t_g, cgr, gr);
                }
                if (!mbar_wait(&u_bar[l % NBU], (l / NBU) & 1, p.status, lim)) failed_sh = 1;
                for (int e = rt; e < C * (DV / 8); e += GR) {  // D U_l as a hi / lo pair
                    const int t = e / (DV / 8), c8 = e % (DV / 8);
                    const uint32_t off = sw128_off(t, c8 * 8, LY::BLK);
                    const uint4 uv = *reinterpret_cast<const uint4 *>(sm + ub + off);
                    const __nv_bfloat16 *hv = reinterpret_cast<const __nv_bfloat16 *>(&uv);
                    float du[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) du[j] = sD[t] * __bfloat162float(hv[j]);
                    uint4 dh, dl;
                    split8(du, dh, dl);
                    st16(sm + LY::DU, off, dh);
                    st16(sm + LY::DUL, off, dl);
                }
                fence_async_smem();
                fence_before_sync();
                named_sync(4, GR);
                fence_after_sync();
                rok = failed_sh == 0;
                if (rok && r_issuer) {
                    const bool acc = l > 0;
                    // [sum P U; O_w] += [P_l; Mqw_l] U_l  (M = 128, accumulated over l)
                    const uint32_t idPU = idesc_bf16(128, DV, 0, 1);
                    mma_steps<C / 16>(tb + LY::cA, idPU, make_desc(sb + LY::P, 16, 1024, 2), dU, ok0, omn, acc);
                    mma_steps<C / 16>(tb + LY::cA, idPU, make_desc(sb + LY::PL, 16, 1024, 2), dU, ok0, omn, true);
                    // F_w += W_l^T [D U_l hi | D U_l lo]  (M = DK: W_l read as an MN-major A operand;
                    // N = 2 DV: the D U tiles sit side by side as one operand)
                    const uint32_t idF = idesc_bf16(DK, 2 * DV, 1, 1);
                    mma_steps<C / 16>(tb + LY::cF, idF, dWmn, make_desc(sb + LY::DU, LY::BLK, 1024, 2), omn, omn, acc);
                    // the next rank's G (its epilogue read of the G columns above is complete)
                    if (l + 1 < L) {
                        if (mbar_wait(&w_bar[(l + 1) & 1], ((l + 1) >> 1) & 1, p.status, lim)) issue_g(l + 1);
                        else failed_sh = 1;
                    }
                }
                rok = r_done(rok);
                // rank l's W and U buffers are free: W_{l+2} and U_{l+NBU} load into them
                if (rok && r_issuer) {
                    if (w_next < L) load_w(w_next++);
                    if (u_next < L) load_u(u_next++);
                }
            }
        }
        // the join: T diag(beta gamma) built, every rank's MMAs complete
        fence_async_smem();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        ok = failed_sh == 0;
        mph = 2 + L;  // G, G_0 and one batch per rank have completed on mma_bar
        // [sum P U; O_w] and F_w read out: the sum P U rows (lane quarters 0-1) become a hi / lo
        // pair over the D U tiles (X_u's operand); O_w (quarters 2-3) is staged over the four
        // [P; Mqw] tiles and F_w (its D U_hi and D U_lo halves summed; row d = lane) over W / U,
        // both in the record's value-slice layout
        if (ok) {
            const int t = 32 * (q & 1) + lane;
#pragma unroll
            for (int cc = hs * (DV / NH); cc < (hs + 1) * (DV / NH); cc += 32) {
                float x[32];
                tmem_ld32(taddr(tb, 32 * q, LY::cA + cc), x);
                tmem_wait_ld();
                if (q < 2) {
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {
                        uint4 hv, lv;
                        split8(x + 8 * c8, hv, lv);
                        const uint32_t off = sw128_off(t, cc + 8 * c8, LY::BLK);
                        st16(sm + LY::DU, off, hv);
                        st16(sm + LY::DUL, off, lv);
                    }
                } else {
#pragma unroll
                    for (int j4 = 0; j4 < 32; j4 += 4) {
                        const int j = cc + j4;
                        *reinterpret_cast<float4 *>(sm + LY::PL + (j / BV) * RC::OW_SLICE + u_off<BV>(t, j % BV)) =
                            make_float4(x[j4], x[j4 + 1], x[j4 + 2], x[j4 + 3]);
                    }
                }
            }
            const int d_row = 32 * q + lane;
#pragma unroll
            for (int cc = hs * (DV / NH); cc < (hs + 1) * (DV / NH); cc += 16) {
                float xh[16], xl[16];
                tmem_ld16(taddr(tb, 32 * q, LY::cF + cc), xh);
                tmem_ld16(taddr(tb, 32 * q, LY::cF + DV + cc), xl);
                tmem_wait_ld();
#pragma unroll
                for (int j4 = 0; j4 < 16; j4 += 4) {
                    const int j = cc + j4;
                    *reinterpret_cast<float4 *>(sm + LY::W + (j / BV) * RC::FW_SLICE + u_off<BV>(d_row, j % BV)) =
                        make_float4(xh[j4] + xl[j4], xh[j4 + 1] + xl[j4 + 1], xh[j4 + 2] + xl[j4 + 2],
                                    xh[j4 + 3] + xl[j4 + 3]);
                }
            }
        }
        fence_async_smem();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        static_assert(RC::FW_SLICE * (DV / BV) <= LY::DU - LY::W, "F_w fits over W and U");
        if (ok && tid == 0) {
            bulk_s2g(rec + RC::OW, sm + LY::PL, C * DV * 4);
            bulk_s2g(rec + RC::FW, sm + LY::W, RC::FW_SLICE * (DV / BV));
            bulk_commit();
            // Wk = T diag(beta gamma) K  (M = 64, into the columns just read out)
            const uint32_t id = idesc_bf16(64, DK, 0, 1);
            mma_steps<C / 16>(tb + LY::cA, id, make_desc(sb + LY::T1, 16, 1024, 2), dKmn, ok0, omn, false);
            mma_steps<C / 16>(tb + LY::cA, id, make_desc(sb + LY::T1L, 16, 1024, 2), dKmn, ok0, omn, true);
        }
        ok = mma_done(ok);
        // Wk as a hi / lo pair staged over K / Q (the Wk MMA was their last reader; hi and lo are
        // adjacent there as WK and WKL in the record), then T itself over the T tiles for X_u
        static_assert(2 * RC::WK_BLK * (DK / 64) <= LY::KQ_BLK * (DK / 64) && LY::BLK == RC::WK_BLK &&
                          RC::WKL == RC::WK + RC::WK_BLK * (DK / 64),
                      "the staged Wk pair has the record's layout");
        if (ok) {
#pragma unroll
            for (int cc = hs * (DK / NH); cc < (hs + 1) * (DK / NH); cc += 32) {
                float x[32];
                tmem_ld32(taddr(tb, 32 * q, LY::cA + cc), x);
                tmem_wait_ld();
                if (own_t) store32_split(sm + LY::KQ, sm + LY::KQ + RC::WK_BLK * (DK / 64), t_row, cc, x, LY::BLK);
            }
            store_t_pair(false, tid, NTH);
        }
        fence_async_smem();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (ok && tid == 0) {
            bulk_s2g(rec + RC::WK, sm + LY::KQ, 2 * RC::WK_BLK * (DK / 64));
            bulk_commit();
            // X_u = T (sum P U)  (M = 64, into the same columns, read out above)
            const uint64_t dPU = make_desc(sb + LY::DU, LY::BLK, 1024, 2);
            const uint64_t dPUL = make_desc(sb + LY::DUL, LY::BLK, 1024, 2);
            const uint64_t dT = make_desc(sb + LY::T1, 16, 1024, 2), dTL = make_desc(sb + LY::T1L, 16, 1024, 2);
            mma_steps<C / 16>(tb + LY::cA, idV, dT, dPU, ok0, omn, false);
            mma_steps<C / 16>(tb + LY::cA, idV, dT, dPUL, ok0, omn, true);
            mma_steps<C / 16>(tb + LY::cA, idV, dTL, dPU, ok0, omn, true);
        }
        ok = mma_done(ok);
        // -X_u -> the U slot, staged over the D U tiles (the X_u MMA was their last reader)
        static_assert((uint32_t)C * DV * 4 <= 2 * LY::BLK * (DK / 64), "-X_u fits over the D U tiles");
        if (ok) {
#pragma unroll
            for (int cc = hs * (DV / NH); cc < (hs + 1) * (DV / NH); cc += 32) {
                float x[32];
                tmem_ld32(taddr(tb, 32 * q, LY::cA + cc), x);
                tmem_wait_ld();
                if (own_t) {
#pragma unroll
                    for (int j4 = 0; j4 < 32; j4 += 4) {
                        const int j = cc + j4;
                        *reinterpret_cast<float4 *>(sm + LY::DU + (j / BV) * RC::U_SLICE + u_off<BV>(t_row, j % BV)) =
                            make_float4(-x[j4], -x[j4 + 1], -x[j4 + 2], -x[j4 + 3]);
                    }
                }
            }
        }
        fence_async_smem();
        fence_before_sync();
        __syncthreads();
        if (ok && tid == 0) {
            bulk_s2g(rec + RC::U, sm + LY::DU, (uint32_t)(C * DV * 4));
            bulk_commit();
        }
        // every bulk store has read its staging before the CTA frees the shared memory; the
        // kernel's end makes the writes visible to the next launch
        if (tid == 0 || r_issuer) bulk_wait_read();
        // after a failure, the rank loop's tile loads still in flight land before the CTA exits
        if (!ok && r_issuer && !stall) {
            for (int l = w_next > 2 ? w_next - 2 : 0; l < w_next; ++l)
                mbar_wait(&w_bar[l & 1], (l >> 1) & 1, nullptr, kStallTestPolls);
            for (int l = u_next > NBU ? u_next - NBU : 0; l < u_next; ++l)
                mbar_wait(&u_bar[l % NBU], (l / NBU) & 1, nullptr, kStallTestPolls);
        }
        w_issued = u_issued = 0;  // (the drain below covers K / Q only)
    }
    // after a failure, let the tile loads still in flight land before the CTA exits
    if (!ok && tid == 0 && !stall) {
        mbar_wait(&ld_bar, 0, nullptr, kStallTestPolls);
        for (int l = w_issued > 2 ? w_issued - 2 : 0; l < w_issued; ++l)
            mbar_wait(&w_bar[l & 1], (l >> 1) & 1, nullptr, kStallTestPolls);
        for (int l = u_issued > NBU ? u_issued - NBU : 0; l < u_issued; ++l)
            mbar_wait(&u_bar[l % NBU], (l / NBU) & 1, nullptr, kStallTestPolls);
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, LY::TCOLS);
}

// ------------------------------------------------------------------------------------------------
// state: one CTA per (value slice, head, batch), chunks in order
//
// Per chunk the chain's MMA thread issues (8 instructions at d = 128 for stage 1, 4 for D4):
//   stage 1:  D1 = [Wk; Q] [S_hi | S_lo]                    (M = 128, N = 2 BV: X_s and QS)
//             D1 += [Wk_lo; *] [S_hi | S_lo], TMEM lanes 64..127 masked off (only X_s gains the
//             Wk_lo term), once the state of this CTA has grown past kBigState
//   D4:       D4 = K^T [DY_hi | DY_lo]                      (the state update)
// and a second thread, in its own warp, the output's intra-chunk term (8 instructions):
//   D3:       D3 = [Mqk_lo; Mqk_hi] [Y_hi | Y_lo], then D3 += [*; Mqk_lo] [Y_hi | Y_lo] with lanes
//             0..63 masked off
// The chain of a chunk is stage 1 -> the Y epilogue -> D4 -> the state epilogue.  One thread
// issues a tcgen05.mma only every 60-80 cycles, so D3 on the chain's thread put its issue time on
// the chain; from its own thread it runs on the tensor pipe while the state epilogue does.  The tile
// Y is double-buffered (D3 of chunk c may still read it while chunk c + 1's Y epilogue runs).
// X_s sits in TMEM lanes 0..63, QS and the whole Mqk Y term in lanes 64..127, so the Y epilogue
// runs on sub-partitions 0-1 and the output epilogue on 2-3.  D1 is double-buffered in TMEM.  K, Q
// arrive by TMA tiled loads, the per-chunk record (Wk, Mqk, the U slice, g, and on the rank-L route
// the F_w slice) by bulk copies, into two chunk buffers: chunk c + 2 loads into chunk c's buffer as
// soon as its readers are done (D4 and the state epilogue's F_w read for most of it, D3 for U and
// Mqk).  Every wait on a barrier that completes once per chunk is made when that barrier can be at
// most one phase ahead of the waiter (parity waits cannot tell two phases apart).
//
// Precision of X_s = Wk S^T: Wk is a rounded intermediate result, so its single-bf16 error (2^-9
// relative) reaches Y scaled by |S|.  For states of order one that stays far below the bf16
// tolerance, but writes with large directions (|w| ~ 8) grow the state into the hundreds.  Each
// CTA therefore watches the largest |S| element of its slice and, once one exceeds kBigState, adds
// the Wk_lo S term (Wk_lo = bf16(Wk - Wk_hi)): the MMA thread loads the next chunk's Wk_lo over
// the Y / D Y tiles (free between a chunk's stage 2 MMAs and the next chunk's Y epilogue) and
// issues 8 more MMAs on the chain at d = 128.

template <int DK, bool RL = false, int BV_ = kBV<DK>>
struct StateLayout {
    static constexpr int BV = BV_;
    static constexpr int N2 = 2 * BV;                     // hi | lo side by side
    // epilogue warps: four per TMEM lane quarter (eight at BV = 16, whose hand-offs then wait for
    // half as many warps; eight columns a thread in both cases but at d = 64)
    static constexpr int EPI = BV == 16 ? 8 : 16;
    static constexpr int CH = BV / (EPI / 4);             // columns of one epilogue warp
    static constexpr int THREADS = 32 * EPI + 96;         // + the chain MMA, load and D3 warps
    // the value tiles (S^T, Y, D Y: [k][hi | lo], MN-major B operands): 64-column blocks with the
    // 128-byte swizzle, or at BV = 16 one 32-column block with the 64-byte swizzle
    static constexpr bool SW64 = N2 == 32;
    static constexpr uint32_t ROWB = SW64 ? 64 : 128;     // bytes of one row of one block
    static constexpr int NBLK = SW64 ? 1 : N2 / 64;
    static constexpr uint32_t VT_SBO = 8 * ROWB;          // stride of 8-row groups
    static constexpr uint32_t VT_LAYOUT = SW64 ? 4 : 2;
    static constexpr uint32_t KWQ_BLK = 3 * C * 128;      // [K; Wk; Q] rows of one 64-col block
    static constexpr uint32_t U_BYTES = C * BV * 4;
    // double-buffered chunk inputs.  U and Mqk are loaded once the buffer's D3 has completed, so
    // the 64 masked rows that D3's second MMA reads in front of Mqk_lo (the end of the U slot,
    // padded to 64 rows of 128 bytes) are not being written while it runs.
    static constexpr uint32_t U_SLOT = U_BYTES >= C * 128 ? U_BYTES : C * 128;
    static constexpr uint32_t B_KWQ = 0;
    static constexpr uint32_t B_U = B_KWQ + KWQ_BLK * (DK / 64);
    static constexpr uint32_t B_MQ = B_U + U_SLOT;                   // [Mqk_lo; Mqk_hi]
    static_assert(B_MQ % 1024 == 0, "the Mqk tile stays 1024-byte aligned");
    static constexpr uint32_t FW_BYTES = RL ? DK * BV * 4 : 0;       // F_w slice (rank L)
    static constexpr uint32_t B_FW = B_MQ + 2 * C * 128;
    static constexpr uint32_t BUF = B_FW + FW_BYTES;
    static_assert(BUF % 1024 == 0, "the second chunk buffer's tiles stay 1024-byte aligned");
    // Y [t][hi | lo] (two buffers, by chunk parity), D Y [t][hi | lo], S^T [d][hi | lo], in the
    // order Y0, D Y, Y1, S.  Wk_lo of chunk c (one 64-row K-major tile per 64 columns) is loaded
    // over D Y and chunk c's Y buffer, which are free from the completion of D4 of chunk c - 1 (the
    // last reader of D Y) and of D3 of chunk c - 2 (the last reader of that Y buffer) to the Y
    // epilogue of chunk c: they are adjacent for either parity.  At BV = 16 those tiles are too
    // small and Wk_lo has a region of its own.
    static constexpr uint32_t Y_BLK = C * ROWB;
    static constexpr uint32_t YT = Y_BLK * NBLK;        // one Y or D Y tile
    static constexpr uint32_t Y0 = 2 * BUF;
    static constexpr uint32_t DY = Y0 + YT;
    static constexpr uint32_t Y1 = DY + YT;
    static constexpr uint32_t WKL_BLK = C * 128;
    static constexpr uint32_t S_BLK = DK * ROWB;
    static constexpr uint32_t S = Y1 + YT;
    // rank L: one O_w slice buffer (the output epilogue's term, loaded a chunk ahead); g of the
    // two chunks in flight
    static constexpr uint32_t OWB = S + S_BLK * NBLK;
    static constexpr uint32_t OW_BYTES = RL ? U_BYTES : 0;
    static constexpr uint32_t GB = OWB + OW_BYTES;
    static constexpr bool WKL_OVER_Y = WKL_BLK * (DK / 64) <= 2 * YT;
    // Wk_lo's own region (with one tile of room for the masked rows past its last block)
    static constexpr uint32_t WKD = (GB + 2 * C * 4 + 1023) / 1024 * 1024;
    static constexpr uint32_t BYTES = (WKL_OVER_Y ? GB + 2 * C * 4 : WKD + WKL_BLK * (DK / 64 + 1)) + 1024;
    static constexpr uint32_t y_at(int c) { return (c & 1) ? Y1 : Y0; }
    static constexpr uint32_t wkl_at(int c) { return WKL_OVER_Y ? ((c & 1) ? DY : Y0) : WKD; }
    // the lane-masked Wk_lo MMA reads 128 rows from each 64-column block of Wk_lo: the rows past
    // the last block (masked, their products dropped) are still inside the allocation
    static_assert(wkl_at(1) + WKL_BLK * (DK / 64) + WKL_BLK <= BYTES - 1024 &&
                      wkl_at(0) + WKL_BLK * (DK / 64) + WKL_BLK <= BYTES - 1024,
                  "masked rows stay in bounds");
    // TMEM columns: D1 (two buffers), D3, D4
    static constexpr uint32_t cD1 = 0, cD3 = 2 * N2, cD4 = 3 * N2;
    static constexpr uint32_t TCOLS = 4 * N2 <= 256 ? 256 : 512;
};

// Warp roles of the state kernel: warps 0 .. EPI-1 epilogue (warp w reads TMEM lane quarter w % 4
// and the column group w / 4 of every BV-wide group), warp EPI issues the chain's MMAs, warp
// EPI + 1 the loads, warp EPI + 2 the D3 MMAs.  Every hand-off is an mbarrier (no CTA-wide barrier
// inside the chunk loop); every wait is bounded.

// Largest |S| element below which X_s = Wk S^T is taken with Wk as one bf16 (its rounding then
// moves Y by at most a few per cent of the bf16 tolerance); above it the Wk_lo term is added.
constexpr float kBigState = 4.0f;
// Output-lane masks of an M = 128 MMA: lanes 64..127 kept as they are, or lanes 0..63.
__device__ __forceinline__ void lane_mask_upper(uint32_t (&m)[4]) {
    m[0] = 0u;
    m[1] = 0u;
    m[2] = 0xffffffffu;
    m[3] = 0xffffffffu;
}
__device__ __forceinline__ void lane_mask_lower(uint32_t (&m)[4]) {
    m[0] = 0xffffffffu;
    m[1] = 0xffffffffu;
    m[2] = 0u;
    m[3] = 0u;
}

struct StateBars {
    uint64_t full[2];      // chunk inputs but U, Mqk landed (tx)
    uint64_t full_mq[2];   // the chunk's U slice and Mqk landed (tx)
    uint64_t empty[2];     // chunk buffer but U, Mqk released: D4 (commit) + every epilogue warp
    uint64_t mq_empty[2];  // the buffer's U, Mqk and Y tile released: that chunk's D3 (commit)
    uint64_t s_ready;      // S^T tile written (every epilogue warp)
    uint64_t y_ready;      // D Y tile written (the warps of lane quarters 0-1)
    uint64_t yq_ready[2];  // Y buffer written (the same warps), by chunk parity
    uint64_t out_free;     // D3 read by the output epilogue (the warps of lane quarters 2-3)
    uint64_t d1_full, d4_full, d3_full;  // MMA -> epilogue: accumulators complete
    uint64_t lo_full;      // Wk_lo of the next chunk landed over Y / D Y (tx)
    uint64_t ow_full;      // rank L: the chunk's O_w slice landed (tx)
    uint64_t ow_read;      // rank L: the O_w slice read (the warps of lane quarters 2-3)
    uint64_t drain, drain3;              // the MMA threads' last operations
};


// CH fp32 values at (row, j0 .. j0+CH) as a hi / lo pair into an MN-major value tile: hi at
// columns j0.., lo at BV + j0...; 64-column 128B-swizzled blocks, or at BV = 16 one 32-column
// 64B-swizzled block (eight columns a thread).
template <int BV, int CH>
__device__ __forceinline__ void store_half_pair(uint8_t *tile, uint32_t blk_bytes, int row, int j0,
                                                const float *x) {
    if constexpr (BV == 16) {
        static_assert(CH == 8, "eight columns a thread of the 32-column tile");
        uint4 hv, lv;
        split8(x, hv, lv);
        st16(tile, sw64_off(row, j0), hv);
        st16(tile, sw64_off(row, BV + j0), lv);
    } else {
#pragma unroll
        for (int c8 = 0; c8 < CH / 8; ++c8) {
            uint4 hv, lv;
            split8(x + c8 * 8, hv, lv);
            st16(tile, sw128_off(row, j0 + c8 * 8, blk_bytes), hv);
            st16(tile, sw128_off(row, BV + j0 + c8 * 8, blk_bytes), lv);
        }
    }
}

template <int DK, bool RL>
__device__ __forceinline__ const uint8_t *record(const ScanArgs &p, const uint8_t *ws, int nch, int c) {
    static_assert(GdnRec<DK, RL, 16>::BYTES == GdnRec<DK, RL>::BYTES, "the record's size does not depend on the slice width");
    return ws + kRecOffset + (((size_t)blockIdx.z * p.H + blockIdx.y) * nch + c) * GdnRec<DK, RL>::BYTES;
}

// One arrival per warp on `bar` once every lane's earlier writes (shared memory, for the tensor
// core) and TMEM reads are complete.
__device__ __forceinline__ void warp_arrive(uint64_t *bar, int lane) {
    fence_async_smem();
    fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar);
}

// CK: also write the entry state of every chunk to ckpt, [B, H, nch, dv, dk] fp32 (the backward's
// checkpoints; a separate instantiation, so the forward's chunk loop carries no test for it).
template <int DK, bool RL, int BV_, bool CK>
__global__ void __launch_bounds__(StateLayout<DK, RL, BV_>::THREADS, 1) gdn_state_kernel(ScanArgs p,
                                                                 const __grid_constant__ GdnMaps maps,
                                                                 const uint8_t *ws, int nch, float *ckpt) {
    using LY = StateLayout<DK, RL, BV_>;
    using RC = GdnRec<DK, RL, BV_>;
    constexpr int BV = LY::BV, N2 = LY::N2, CH = LY::CH, EPI_WARPS = LY::EPI;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ StateBars bars;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int failed_sh;
    __shared__ int big_sh;  // set once some |S| element of this slice exceeds kBigState

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int v0 = blockIdx.x * BV, h = blockIdx.y, b = blockIdx.z;
    const int H = p.H, T = p.T, dv = p.dv;
    const size_t head = (size_t)b * H + h;
    const uint32_t sb = smem_u32(sm);

    if (warp == 0) tmem_alloc(&tmem_base_sh, LY::TCOLS);
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars.full[i], 1);
            mbar_init(&bars.full_mq[i], 1);
            mbar_init(&bars.empty[i], 1 + EPI_WARPS);
            mbar_init(&bars.mq_empty[i], 1);
        }
        mbar_init(&bars.s_ready, EPI_WARPS);
        mbar_init(&bars.y_ready, EPI_WARPS / 2);
        mbar_init(&bars.yq_ready[0], EPI_WARPS / 2);
        mbar_init(&bars.yq_ready[1], EPI_WARPS / 2);
        mbar_init(&bars.out_free, EPI_WARPS / 2);
        mbar_init(&bars.d1_full, 1);
        mbar_init(&bars.d4_full, 1);
        mbar_init(&bars.d3_full, 1);
        mbar_init(&bars.lo_full, 1);
        mbar_init(&bars.ow_full, 1);
        mbar_init(&bars.ow_read, EPI_WARPS / 2);
        mbar_init(&bars.drain, 1);
        mbar_init(&bars.drain3, 1);
        mbar_fence_init();
        failed_sh = 0;
        big_sh = (p.flags & kForceWkLo) ? 1 : 0;
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tb = tmem_base_sh;
    uint32_t *status = p.status;
    const uint32_t lim = (p.flags & kStallTest) ? kStallTestPolls : kWaitPolls;
    auto fail = [&]() { failed_sh = 1; };
    auto failed = [&]() { return *(volatile int *)&failed_sh != 0; };

    if (warp == EPI_WARPS + 1) {
        // ---------------- loads ----------------
        if (lane == 0) {
            constexpr uint32_t bytes = 3 * (DK / 64) * C * 128 + C * 4 + LY::FW_BYTES;
            constexpr uint32_t bytes_mq = LY::U_BYTES + 2 * C * 128;
            int issued = -1, issued_mq = -1;
            for (int c = 0; c < nch && !failed() && !(p.flags & kStallTest); ++c) {
                // the buffer's main part frees after D4 of chunk c - 2, its U and Mqk after that
                // chunk's D3 (the Y epilogue read U before the epilogue warps released the buffer)
                if (c >= 2 && !mbar_wait(&bars.empty[c & 1], ((c - 2) >> 1) & 1, status, lim)) { fail(); break; }
                const uint8_t *rec = record<DK, RL>(p, ws, nch, c);
                uint8_t *buf = sm + (c & 1) * LY::BUF;
                uint64_t *bar = &bars.full[c & 1];
                const int c0 = c * C;
                mbar_expect_tx(bar, bytes);
                for (int blk = 0; blk < DK / 64; ++blk) {
                    uint8_t *dst = buf + LY::B_KWQ + blk * LY::KWQ_BLK;
                    tma_load_4d(dst, &maps.k, blk * 64, h, c0, b, bar);
                    bulk_g2s(dst + C * 128, rec + RC::WK + blk * RC::WK_BLK, RC::WK_BLK, bar);
                    tma_load_4d(dst + 2 * C * 128, &maps.q, blk * 64, h, c0, b, bar);
                }
                // once the state is large the MMA thread loads this chunk's Wk_lo: start it to L2
                if (*(volatile int *)&big_sh) bulk_prefetch_l2(rec + RC::WKL, RC::WK_BLK * (DK / 64));
                bulk_g2s(sm + LY::GB + (c & 1) * C * 4, rec + RC::G, C * 4, bar);
                if constexpr (RL)
                    bulk_g2s(buf + LY::B_FW, rec + RC::FW + blockIdx.x * RC::FW_SLICE, LY::FW_BYTES, bar);
                issued = c;
                if (c >= 2 && !mbar_wait(&bars.mq_empty[c & 1], ((c - 2) >> 1) & 1, status, lim)) { fail(); break; }
                uint64_t *bar_mq = &bars.full_mq[c & 1];
                mbar_expect_tx(bar_mq, bytes_mq);
                bulk_g2s(buf + LY::B_U, rec + RC::U + blockIdx.x * RC::U_SLICE, LY::U_BYTES, bar_mq);
                bulk_g2s(buf + LY::B_MQ, rec + RC::MQK + C * 128, C * 128, bar_mq);   // Mqk_lo
                bulk_g2s(buf + LY::B_MQ + C * 128, rec + RC::MQK, C * 128, bar_mq);   // Mqk_hi
                issued_mq = c;
            }
            // let the copies still in flight land before the CTA can exit
            for (int c = issued > 0 ? issued - 1 : 0; c <= issued; ++c)
                mbar_wait(&bars.full[c & 1], (c >> 1) & 1, nullptr, lim);
            for (int c = issued_mq > 0 ? issued_mq - 1 : 0; c <= issued_mq; ++c)
                mbar_wait(&bars.full_mq[c & 1], (c >> 1) & 1, nullptr, lim);
        }
    } else if (warp == EPI_WARPS + 2) {
        // ---------------- D3 MMA issue ----------------
        if (lane == 0) {
            auto oK0 = [](int ks) { return (uint64_t)koff_k_sw128(ks, 0); };
            auto oVT = [](int ks) { return (uint64_t)(LY::SW64 ? koff_mn_sw64(ks) : koff_mn_sw128(ks)); };
            const uint32_t idS = idesc_bf16(128, N2, 0, 1);
            uint32_t omask[4];
            lane_mask_lower(omask);  // the Mqk_lo output term: output rows only (lanes 64..127)
            bool ok = true;
            for (int c = 0; c < nch && ok; ++c) {
                // D3 of chunk c: Mqk Y for the output rows (lanes 64..127).  [Mqk_lo; Mqk_hi] Y puts
                // the Mqk_hi rows there, then [Q rows; Mqk_lo] Y adds the Mqk_lo rows with lanes
                // 0..63 masked.  It waits for Y_c, the chunk's U / Mqk, and the output epilogue's
                // read of D3 of chunk c - 1.
                if (!mbar_wait(&bars.yq_ready[c & 1], (c >> 1) & 1, status, lim) ||
                    !mbar_wait(&bars.full_mq[c & 1], (c >> 1) & 1, status, lim) ||
                    (c > 0 && !mbar_wait(&bars.out_free, (c - 1) & 1, status, lim))) {
                    ok = false;
                    break;
                }
                fence_after_sync();
                const uint32_t bb = sb + (c & 1) * LY::BUF;
                const uint64_t dY2 = make_desc(sb + LY::y_at(c), LY::SW64 ? 0 : LY::Y_BLK, LY::VT_SBO, LY::VT_LAYOUT);
                mma_steps<C / 16>(tb + LY::cD3, idS, make_desc(bb + LY::B_MQ, 16, 1024, 2), dY2, oK0, oVT, false);
                mma_steps_lanes<C / 16>(tb + LY::cD3, idS, make_desc(bb + LY::B_MQ - C * 128, 16, 1024, 2), dY2,
                                        oK0, oVT, true, omask);
                mma_commit(&bars.d3_full);
                mma_commit(&bars.mq_empty[c & 1]);
            }
            if (!ok) fail();
            mma_commit(&bars.drain3);
            mbar_wait(&bars.drain3, 0, nullptr, lim);
        }
    } else if (warp == EPI_WARPS) {
        // ---------------- chain MMA issue ----------------
        if (lane == 0) {
            auto oKWQ = [](int ks) { return (uint64_t)koff_k_sw128(ks, LY::KWQ_BLK); };
            auto oMN = [](int ks) { return (uint64_t)koff_mn_sw128(ks); };  // K^T (the K tile)
            auto oVT = [](int ks) { return (uint64_t)(LY::SW64 ? koff_mn_sw64(ks) : koff_mn_sw128(ks)); };
            const uint64_t dS2 = make_desc(sb + LY::S, LY::SW64 ? 0 : LY::S_BLK, LY::VT_SBO, LY::VT_LAYOUT);
            const uint64_t dDY2 = make_desc(sb + LY::DY, LY::SW64 ? 0 : LY::Y_BLK, LY::VT_SBO, LY::VT_LAYOUT);
            const uint32_t idS = idesc_bf16(128, N2, 0, 1);
            const uint32_t id4 = idesc_bf16(DK, N2, 1, 1);
            auto oLO = [](int ks) { return (uint64_t)koff_k_sw128(ks, LY::WKL_BLK); };
            uint32_t xmask[4];
            lane_mask_upper(xmask);  // the Wk_lo term: X_s rows only (lanes 64..127 hold Q S)
            // Wk_lo of chunk c over D Y and Y buffer c % 2 (bulk copies; lo_full counts its bytes)
            uint32_t lo_phase = 0;
            auto load_lo = [&](int c) {
                const uint8_t *rec = record<DK, RL>(p, ws, nch, c);
                mbar_expect_tx(&bars.lo_full, LY::WKL_BLK * (DK / 64));
                for (int blk = 0; blk < DK / 64; ++blk)
                    bulk_g2s(sm + LY::wkl_at(c) + blk * LY::WKL_BLK, rec + RC::WKL + blk * RC::WK_BLK,
                             RC::WK_BLK, &bars.lo_full);
            };
            bool lo = false;  // this chunk's Wk_lo is loaded (or on its way)
            if (nch > 0 && *(volatile int *)&big_sh) {
                load_lo(0);
                lo = true;
            }
            bool ok = nch == 0 || mbar_wait(&bars.full[0], 0, status, lim);
            for (int c = 0; c < nch && ok; ++c) {
                const uint32_t bb = sb + (c & 1) * LY::BUF;
                // S_c written (which also means every epilogue read of this D1 buffer, two chunks
                // back, is done: the epilogue warps work through the chunks in order)
                if (!mbar_wait_spin(&bars.s_ready, c & 1, status, lim)) { ok = false; break; }
                fence_after_sync();
                const uint64_t dWQ = make_desc(bb + LY::B_KWQ + C * 128, 16, 1024, 2);
                mma_steps<DK / 16>(tb + LY::cD1 + (c & 1) * N2, idS, dWQ, dS2, oKWQ, oVT, false);
                // S_c turned out large after the prefetch decision for this chunk was taken: its
                // Wk_lo is loaded now (once per CTA; every later chunk's is prefetched).  The region
                // is free: D4 of chunk c - 1 has completed (S_c was written after it), and D3 of
                // chunk c - 2, the last reader of Y buffer c % 2, is waited for.
                if (!lo && *(volatile int *)&big_sh) {
                    if (LY::WKL_OVER_Y && c >= 2 &&
                        !mbar_wait(&bars.mq_empty[c & 1], ((c - 2) >> 1) & 1, status, lim)) {
                        ok = false;
                        break;
                    }
                    load_lo(c);
                    lo = true;
                }
                if (lo) {  // X_s += Wk_lo S, into the same accumulator with the Q S rows masked
                    if (!mbar_wait(&bars.lo_full, lo_phase & 1, status, lim)) { ok = false; break; }
                    ++lo_phase;
                    const uint64_t dLW = make_desc(sb + LY::wkl_at(c), 16, 1024, 2);
                    mma_steps_lanes<DK / 16>(tb + LY::cD1 + (c & 1) * N2, idS, dLW, dS2, oLO, oVT, true, xmask);
                    lo = false;
                }
                mma_commit(&bars.d1_full);
                // D Y_c written
                if (!mbar_wait_spin(&bars.y_ready, c & 1, status, lim)) { ok = false; break; }
                fence_after_sync();
                const uint64_t dKt = make_desc(bb + LY::B_KWQ, LY::KWQ_BLK, 1024, 2);
                mma_steps<C / 16>(tb + LY::cD4, id4, dKt, dDY2, oMN, oVT, false);
                mma_commit(&bars.d4_full);
                mma_commit(&bars.empty[c & 1]);
                if (c + 1 < nch) {
                    // once the state is large: the next chunk's Wk_lo over D Y and Y buffer
                    // (c + 1) % 2, as soon as D4 of chunk c and D3 of chunk c - 1 have completed
                    // (the latter cannot be a phase further on: D3 of chunk c + 1 needs this Wk_lo)
                    if (*(volatile int *)&big_sh) {
                        if (!mbar_wait(&bars.d4_full, c & 1, status, lim) ||
                            (c >= 1 && !mbar_wait(&bars.mq_empty[(c + 1) & 1], ((c - 1) >> 1) & 1, status, lim))) {
                            ok = false;
                            break;
                        }
                        load_lo(c + 1);
                        lo = true;
                    }
                    // the next chunk's inputs, off the chain while the state epilogue runs
                    if (!mbar_wait(&bars.full[(c + 1) & 1], ((c + 1) >> 1) & 1, status, lim)) { ok = false; break; }
                }
            }
            if (!ok) fail();
            mma_commit(&bars.drain);
            mbar_wait(&bars.drain, 0, nullptr, lim);
            if (lo) mbar_wait(&bars.lo_full, lo_phase & 1, nullptr, lim);  // a copy still in flight lands
        }
    } else {
        // ---------------- epilogue: warps 0-15 ----------------
        __nv_bfloat16 *o = (__nv_bfloat16 *)p.o;
        const int q = warp & 3;            // TMEM lane quarter
        const int j0 = (warp >> 2) * CH;   // first column of this warp in each BV-wide group
        const int lrow = 32 * q + lane;    // TMEM lane of this thread
        const bool lowq = q < 2;           // lanes 0..63: X_s -> Y; lanes 64..127: the output rows
        // state rows: lane = row for M = 128 (d = 128); lanes 32q + r, r < 16, for M = 64
        const bool own_d = (DK == 128) ? true : (lane < 16);
        const int d_row = (DK == 128) ? lrow : (16 * q + lane);
        const bool wr = !(p.flags & kNoWrite), out = !(p.flags & kNoOutput);
        float Sreg[CH];
#pragma unroll
        for (int j = 0; j < CH; ++j) Sreg[j] = 0.f;
        if (own_d && (p.flags & kS0Identity)) {
#pragma unroll
            for (int j = 0; j < CH; ++j) Sreg[j] = (v0 + j0 + j == d_row) ? 1.f : 0.f;
        } else if (own_d && p.S0) {
#pragma unroll
            for (int j = 0; j < CH; ++j) Sreg[j] = p.S0[(head * dv + v0 + j0 + j) * DK + d_row];
        }
        // the Wk_lo switch: set (never cleared) once an element of this slice's state is large
        auto watch_state = [&]() {
            float m = 0.f;
#pragma unroll
            for (int j = 0; j < CH; ++j) m = fmaxf(m, fabsf(Sreg[j]));
            if (m > kBigState) big_sh = 1;
        };
        // rank L: the output's O_w term arrives in one shared-memory slice buffer by a bulk copy
        // that the first output-row thread issues once every output warp has read the previous
        // chunk's slice (ow_read), a chunk ahead of its use
        const bool ow_on = RL && wr && out;
        const bool ow_issuer = tid == 64;  // warp 2, lane 0 (lane quarter 2)
        int ow_issued = 0, ow_seen = 0;
        auto load_ow = [&](int c) {
            if constexpr (RL) {
                mbar_expect_tx(&bars.ow_full, LY::OW_BYTES);
                bulk_g2s(sm + LY::OWB, record<DK, RL>(p, ws, nch, c) + RC::OW + blockIdx.x * RC::OW_SLICE,
                         LY::OW_BYTES, &bars.ow_full);
                ++ow_issued;
            }
        };
        if (ow_on && ow_issuer && nch > 0) load_ow(0);
        if (own_d) {
            store_half_pair<BV, CH>(sm + LY::S, LY::S_BLK, d_row, j0, Sreg);
            watch_state();
        }
        warp_arrive(&bars.s_ready, lane);
        bool ok = true;
        for (int c = 0; c < nch && ok; ++c) {
            const int c0 = c * C, n = min(C, T - c0);
            const uint8_t *buf = sm + (c & 1) * LY::BUF;
            if (CK && own_d) {  // the chunk's entry state, for the backward
                float *ck = ckpt + ((head * nch + c) * dv + v0 + j0) * DK + d_row;
#pragma unroll
                for (int j = 0; j < CH; ++j) ck[(size_t)j * DK] = Sreg[j];
            }
            if (!mbar_wait(&bars.full[c & 1], (c >> 1) & 1, status, lim)) { ok = false; break; }
            const float *g = reinterpret_cast<const float *>(sm + LY::GB + (c & 1) * C * 4);
            const float g_last = g[C - 1];
            const float g_row = g[lowq ? lrow : lrow - 64];  // g of this thread's Y / output row
            const uint32_t d1 = LY::cD1 + (c & 1) * N2;
            // Y = U - X_s (lanes 0..63 of D1), and D Y: D Y first (D4 waits for it), Y after the
            // hand-off (D3 reads it after the next state hand-off)
            if (lowq) {
                const int t = lrow;
                const float dd = t < n ? __expf(g_last - g_row) : 0.f;
                if (!mbar_wait(&bars.full_mq[c & 1], (c >> 1) & 1, status, lim)) { ok = false; break; }
                float y[CH];  // U first: it does not depend on D1
#pragma unroll
                for (int j4 = 0; j4 < CH; j4 += 4) {
                    const float4 u = wr ? *reinterpret_cast<const float4 *>(buf + LY::B_U + u_off<BV>(t, j0 + j4))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                    y[j4] = u.x;
                    y[j4 + 1] = u.y;
                    y[j4 + 2] = u.z;
                    y[j4 + 3] = u.w;
                }
                if (!mbar_wait(&bars.d1_full, c & 1, status, lim)) { ok = false; break; }
                fence_after_sync();
                float xh[CH], xl[CH];
                tmem_ld_n<CH>(taddr(tb, 32 * q, d1 + j0), xh);
                tmem_ld_n<CH>(taddr(tb, 32 * q, d1 + BV + j0), xl);
                tmem_wait_ld();
                float dy[CH];
#pragma unroll
                for (int j = 0; j < CH; ++j) {
                    y[j] -= xh[j] + xl[j];
                    dy[j] = y[j] * dd;
                }
                store_half_pair<BV, CH>(sm + LY::DY, LY::Y_BLK, t, j0, dy);
                warp_arrive(&bars.y_ready, lane);
                // Y buffer c % 2 was last read by D3 of chunk c - 2, which has completed: the output
                // warps saw it complete before they wrote S_c, and this chunk's stage 1, whose
                // completion these warps saw, was issued after S_c
                store_half_pair<BV, CH>(sm + LY::y_at(c), LY::Y_BLK, t, j0, y);
                warp_arrive(&bars.yq_ready[c & 1], lane);
            }
            // state update S^T <- e^{g_n} S^T + K^T D Y (+ F_w)
            {
                const float gC = __expf(g_last);
                if (own_d) {  // e^{g_n} S^T (+ F_w): no D4 needed yet
#pragma unroll
                    for (int j = 0; j < CH; ++j) Sreg[j] *= gC;
                    if (RL && wr) {
#pragma unroll
                        for (int j4 = 0; j4 < CH; j4 += 4) {
                            const float4 f4 = *reinterpret_cast<const float4 *>(buf + LY::B_FW + u_off<BV>(d_row, j0 + j4));
                            Sreg[j4] += f4.x;
                            Sreg[j4 + 1] += f4.y;
                            Sreg[j4 + 2] += f4.z;
                            Sreg[j4 + 3] += f4.w;
                        }
                    }
                }
                // the last read of the chunk buffer (g is held in registers): release it, so that
                // the chunk two ahead loads while this one's state and output epilogues run
                warp_arrive(&bars.empty[c & 1], lane);
                if (!mbar_wait(&bars.d4_full, c & 1, status, lim)) { ok = false; break; }
                fence_after_sync();
                float xh[CH], xl[CH];
                tmem_ld_n<CH>(taddr(tb, 32 * q, LY::cD4 + j0), xh);
                tmem_ld_n<CH>(taddr(tb, 32 * q, LY::cD4 + BV + j0), xl);
                tmem_wait_ld();
                if (own_d) {
                    float m[2] = {0.f, 0.f};  // the size check of S_{c+1} (two independent chains)
#pragma unroll
                    for (int j = 0; j < CH; ++j) {
                        Sreg[j] += xh[j] + xl[j];
                        m[j & 1] = fmaxf(m[j & 1], fabsf(Sreg[j]));
                    }
                    store_half_pair<BV, CH>(sm + LY::S, LY::S_BLK, d_row, j0, Sreg);
                    if (fmaxf(m[0], m[1]) > kBigState) big_sh = 1;
                }
            }
            warp_arrive(&bars.s_ready, lane);
            // output O = diag(e^g) QS + Mqk Y (+ O_w), by the threads of the output rows (TMEM lanes
            // 64..127, where both the Q S rows of D1 and the whole Mqk Y term of D3 sit)
            if (!lowq) {
                if (!mbar_wait(&bars.d3_full, c & 1, status, lim)) { ok = false; break; }
                fence_after_sync();
                const int t = lrow - 64;
                float up[CH], qs[CH];
                {
                    float a[CH], bb[CH];
                    tmem_ld_n<CH>(taddr(tb, 32 * q, LY::cD3 + j0), a);
                    tmem_ld_n<CH>(taddr(tb, 32 * q, LY::cD3 + BV + j0), bb);
                    tmem_wait_ld();
                    warp_arrive(&bars.out_free, lane);  // D3 may be overwritten by the next chunk's
#pragma unroll
                    for (int j = 0; j < CH; ++j) up[j] = a[j] + bb[j];
                    tmem_ld_n<CH>(taddr(tb, 32 * q, d1 + j0), a);
                    tmem_ld_n<CH>(taddr(tb, 32 * q, d1 + BV + j0), bb);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < CH; ++j) qs[j] = a[j] + bb[j];
                }
                float ow[CH];  // rank L: O_w of this thread's row
#pragma unroll
                for (int j = 0; j < CH; ++j) ow[j] = 0.f;
                if (ow_on) {
                    if (!mbar_wait(&bars.ow_full, c & 1, status, lim)) { ok = false; break; }
                    ++ow_seen;
                    if (t < n) {
#pragma unroll
                        for (int j4 = 0; j4 < CH; j4 += 4) {
                            const float4 f4 = *reinterpret_cast<const float4 *>(sm + LY::OWB + u_off<BV>(t, j0 + j4));
                            ow[j4] = f4.x;
                            ow[j4 + 1] = f4.y;
                            ow[j4 + 2] = f4.z;
                            ow[j4 + 3] = f4.w;
                        }
                    }
                    warp_arrive(&bars.ow_read, lane);
                }
                if (t < n && out) {
                    const float gt = __expf(g_row);
                    __nv_bfloat16 *dst = o + (((size_t)b * T + c0 + t) * H + h) * dv + v0 + j0;
#pragma unroll
                    for (int c8 = 0; c8 < CH / 8; ++c8) {
                        float r[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int jj = c8 * 8 + j;
                            r[j] = fmaf(gt, qs[jj], up[jj] + ow[jj]);
                        }
                        uint4 pk;
                        pk.x = pack_bf16(r[0], r[1]);
                        pk.y = pack_bf16(r[2], r[3]);
                        pk.z = pack_bf16(r[4], r[5]);
                        pk.w = pack_bf16(r[6], r[7]);
                        *reinterpret_cast<uint4 *>(dst + c8 * 8) = pk;
                    }
                }
                // the next chunk's O_w slice, once every output warp has read this one
                if (ow_on && ow_issuer && c + 1 < nch) {
                    if (!mbar_wait(&bars.ow_read, c & 1, status, lim)) { ok = false; break; }
                    load_ow(c + 1);
                }
            }
        }
        if (!ok) fail();
        // a copy still in flight (the loop stopped early) lands before the CTA exits
        if (ow_issuer && ow_issued > ow_seen) mbar_wait(&bars.ow_full, (ow_issued - 1) & 1, nullptr, lim);
        if (p.S_final && own_d && !failed()) {
#pragma unroll
            for (int j = 0; j < CH; ++j) p.S_final[(head * dv + v0 + j0 + j) * DK + d_row] = Sreg[j];
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

template <int DK>
bool gdn_maps(const ScanArgs &a, GdnMaps *maps) {
    return act_map(&maps->k, a.k, a.B, a.T, a.H, DK, 64) && act_map(&maps->q, a.q, a.B, a.T, a.H, DK, 64) &&
           act_map(&maps->v, a.v, a.B, a.T, a.H, a.dv, 64);
}

// Host: the SM count of the current device (cached per device).
int device_sms() {
    static int sms[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        sms[dev] = n;
    }
    return sms[dev];
}

// Value-slice width of the state kernel, and of the record's slice-major parts, which the prep
// writes to match (both take it from the same shape): 16 at d = 128 when 16-wide slices still
// give every in-order chain an SM of its own (few sequences: each chain then moves half the value
// columns per chunk through its SM's shared memory, on twice as many SMs), else kBV.
template <int DK>
int slice_width(const ScanArgs &a) {
    if (DK != 128) return kBV<DK>;
    const long long chains = (long long)a.B * a.H * (a.dv / 16);
    return chains <= device_sms() ? 16 : kBV<DK>;
}

template <int DK, int BV>
cudaError_t launch_gdn_prep_bv(const ScanArgs &a, void *ws, cudaStream_t s) {
    const int nch = (a.T + C - 1) / C;
    GdnMaps maps;
    if (!gdn_maps<DK>(a, &maps)) return cudaErrorInvalidValue;
    using LY = PrepLayout<DK>;
    auto kern = gdn_prep_kernel<DK, BV>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)LY::BYTES);
    if (err != cudaSuccess) return err;
    dim3 grid(nch, a.H, a.B);
    launch_probe_mark(s);
    kern<<<grid, PREP_THREADS, LY::BYTES, s>>>(a, maps, (uint8_t *)ws, nch);
    return cudaGetLastError();
}

template <int DK>
cudaError_t launch_gdn_prep_t(const ScanArgs &a, void *ws, cudaStream_t s) {
    if constexpr (DK == 128)
        if (slice_width<DK>(a) == 16) return launch_gdn_prep_bv<DK, 16>(a, ws, s);
    return launch_gdn_prep_bv<DK, kBV<DK>>(a, ws, s);
}

// The state kernel reads only K and Q through tensor maps (v may be absent on the rank-L route).
template <int DK, bool RL, int BV>
cudaError_t launch_gdn_state_bv(const ScanArgs &a, const void *ws, cudaStream_t s, float *ckpt) {
    const int nch = (a.T + C - 1) / C;
    GdnMaps maps = {};
    if (!act_map(&maps.k, a.k, a.B, a.T, a.H, DK, 64) || !act_map(&maps.q, a.q, a.B, a.T, a.H, DK, 64))
        return cudaErrorInvalidValue;
    using LY = StateLayout<DK, RL, BV>;
    static_assert(LY::BYTES + 256 <= 227 * 1024, "shared memory budget (with the static part)");
    auto kern = ckpt ? gdn_state_kernel<DK, RL, BV, true> : gdn_state_kernel<DK, RL, BV, false>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)LY::BYTES);
    if (err != cudaSuccess) return err;
    dim3 grid(a.dv / LY::BV, a.H, a.B);
    launch_probe_mark(s);
    kern<<<grid, LY::THREADS, LY::BYTES, s>>>(a, maps, (const uint8_t *)ws, nch, ckpt);
    return cudaGetLastError();
}

template <int DK, bool RL>
cudaError_t launch_gdn_state_t(const ScanArgs &a, const void *ws, cudaStream_t s, float *ckpt) {
    if constexpr (DK == 128)
        if (slice_width<DK>(a) == 16) return launch_gdn_state_bv<DK, RL, 16>(a, ws, s, ckpt);
    return launch_gdn_state_bv<DK, RL, kBV<DK>>(a, ws, s, ckpt);
}

template <int DK, int BV>
cudaError_t launch_lrank_prep_bv(const ScanArgs &a, void *ws, cudaStream_t s) {
    const int nch = (a.T + C - 1) / C;
    LMaps maps;
    if (!act_map(&maps.k, a.k, a.B, a.T, a.H, DK, 64) || !act_map(&maps.q, a.q, a.B, a.T, a.H, DK, 64) ||
        !act_map(&maps.w, a.w, a.B, a.T, a.H * a.L, DK, 64) ||
        !act_map(&maps.u, a.u, a.B, a.T, a.H * a.L, a.dv, 64))
        return cudaErrorInvalidValue;
    using LY = LPrepLayout<DK>;
    static_assert(LY::BYTES <= 227 * 1024, "shared memory budget");
    auto kern = lrank_prep_kernel<DK, BV>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)LY::BYTES);
    if (err != cudaSuccess) return err;
    dim3 grid(nch, a.H, a.B);
    launch_probe_mark(s);
    kern<<<grid, kLPrepThreads<DK>, LY::BYTES, s>>>(a, maps, (uint8_t *)ws, nch);
    return cudaGetLastError();
}

template <int DK>
cudaError_t launch_lrank_prep_t(const ScanArgs &a, void *ws, cudaStream_t s) {
    if constexpr (DK == 128)
        if (slice_width<DK>(a) == 16) return launch_lrank_prep_bv<DK, 16>(a, ws, s);
    return launch_lrank_prep_bv<DK, kBV<DK>>(a, ws, s);
}

}  // namespace

// Workspace bytes of the two-kernel path: the status block plus one record per chunk.
size_t gdn_workspace_bytes(int B, int H, int T, int dk) {
    const size_t nch = (size_t)((T + C - 1) / C);
    const size_t rec = dk == 128 ? GdnRec<128>::BYTES : GdnRec<64>::BYTES;
    return kRecOffset + (size_t)B * H * nch * rec;
}
size_t lrank_workspace_bytes(int B, int H, int T, int dk) {
    const size_t nch = (size_t)((T + C - 1) / C);
    const size_t rec = dk == 128 ? GdnRec<128, true>::BYTES : GdnRec<64, true>::BYTES;
    return kRecOffset + (size_t)B * H * nch * rec;
}

// The per-chunk records (prep) and the in-order pass over them (state); records depend only on
// the tokens (q, k, v, alpha, beta), so several state passes over the same tokens can share one
// prep (a pass with kNoWrite ignores the records' U).
cudaError_t launch_gdn_prep(const ScanArgs &a, void *ws, cudaStream_t s) {
    if (a.T <= 0) return cudaSuccess;
    return a.dk == 128 ? launch_gdn_prep_t<128>(a, ws, s) : launch_gdn_prep_t<64>(a, ws, s);
}

// ckpt (optional): every chunk's entry state, [B, H, ceil(T / 64), dv, dk] fp32
cudaError_t launch_gdn_state(const ScanArgs &a, const void *ws, cudaStream_t s, float *ckpt) {
    return a.dk == 128 ? launch_gdn_state_t<128, false>(a, ws, s, ckpt) : launch_gdn_state_t<64, false>(a, ws, s, ckpt);
}
cudaError_t launch_gdn_state(const ScanArgs &a, const void *ws, cudaStream_t s) { return launch_gdn_state(a, ws, s, nullptr); }

cudaError_t launch_scan_gdn(const ScanArgs &a, void *ws, cudaStream_t s) {
    cudaError_t err = launch_gdn_prep(a, ws, s);
    if (err != cudaSuccess) return err;
    return launch_gdn_state(a, ws, s);
}

// The rank-L write on the same two-kernel schedule: the records add O_w and F_w, and their U slot
// holds -X_u.  Requires bf16 I/O, dk == dv in {64, 128}, 1 <= L <= 8.
cudaError_t launch_lrank_prep(const ScanArgs &a, void *ws, cudaStream_t s) {
    if (a.T <= 0) return cudaSuccess;
    return a.dk == 128 ? launch_lrank_prep_t<128>(a, ws, s) : launch_lrank_prep_t<64>(a, ws, s);
}

cudaError_t launch_lrank_state(const ScanArgs &a, const void *ws, cudaStream_t s, float *ckpt) {
    return a.dk == 128 ? launch_gdn_state_t<128, true>(a, ws, s, ckpt) : launch_gdn_state_t<64, true>(a, ws, s, ckpt);
}
cudaError_t launch_lrank_state(const ScanArgs &a, const void *ws, cudaStream_t s) { return launch_lrank_state(a, ws, s, nullptr); }

cudaError_t launch_scan_lrank(const ScanArgs &a, void *ws, cudaStream_t s) {
    cudaError_t err = launch_lrank_prep(a, ws, s);
    if (err != cudaSuccess) return err;
    return launch_lrank_state(a, ws, s);
}

}  // namespace prism
