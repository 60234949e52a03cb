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
// One CTA per 128 tokens of one (batch, head), two CTAs per SM at d = 64: eight epilogue warps build the anchor tile (the A
// operand, as a bf16 hi / lo pair: a single bf16 anchor lets the residual chain amplify its
// rounding past the bf16 output tolerance by the fourth rank) and hold the residual in registers (a token row and half its columns a thread);
// one warp loads the weights by TMA (double-buffered per l) and issues, for each l, one
// M = 128, N = 2d MMA into one of two TMEM accumulators, so the MMA of rank l + 1 runs while the
// epilogue of rank l reads k^(l) and p^(l), applies the GELU step and stores u and w.  Every wait
// is a bounded mbarrier poll that records PRISM_ERR_TIMEOUT in the library's producer status word.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "chunk_common.cuh"
#include "producer.cuh"

namespace prism {
namespace {

__device__ uint32_t g_producer_status;

constexpr int PT = 128;                    // tokens per CTA (TMEM lanes, M of the MMA)
constexpr int P_EPI = 8;                   // epilogue warps
constexpr int P_THREADS = 32 * (P_EPI + 1);
constexpr float kRsqrt2 = 0.70710678118654752f;

template <int D>
struct ProdLayout {
    static constexpr uint32_t A_BLK = PT * 128;            // 128 token rows x 64 bf16 columns
    static constexpr uint32_t A = 0;                       // anchor hi tile, K-major SW128
    static constexpr uint32_t A_LO = A + A_BLK * (D / 64); // anchor lo tile
    static constexpr uint32_t W_BLK = 2 * D * 128;         // [W_k; W_p] rows of one 64-col block
    static constexpr uint32_t WBUF = W_BLK * (D / 64);
    static constexpr uint32_t W = A_LO + A_BLK * (D / 64); // two weight buffers
    static constexpr uint32_t BYTES = W + 2 * WBUF + 1024;
    static constexpr uint32_t TCOLS = 4 * D <= 256 ? 256 : 512;   // two [k | p] accumulators
    static_assert(BYTES <= 227 * 1024, "shared memory budget");
};

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

template <int D>
__global__ void __launch_bounds__(P_THREADS, D == 64 ? 2 : 1) write_producer_kernel(ProducerArgs p,
                                                                     const __grid_constant__ CUtensorMap mk,
                                                                     const __grid_constant__ CUtensorMap mp) {
    using LY = ProdLayout<D>;
    constexpr int HALF = D / 2;  // columns of an epilogue thread
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t wbar[2], full[2], tfree[2], a_ready, drain;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int failed_sh;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = blockIdx.x * PT, h = blockIdx.y, b = blockIdx.z;
    const int T = p.T, H = p.H, L = p.L;
    const uint32_t sb = smem_u32(sm);
    uint32_t *status = &g_producer_status;
    const uint32_t lim = p.stall ? kStallTestPolls : kWaitPolls;

    if (warp == P_EPI) tmem_alloc(&tmem_base_sh, LY::TCOLS);
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&wbar[i], 1);
            mbar_init(&full[i], 1);
            mbar_init(&tfree[i], P_EPI);
        }
        mbar_init(&a_ready, P_EPI);
        mbar_init(&drain, 1);
        mbar_fence_init();
        failed_sh = 0;
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tb = tmem_base_sh;

    if (warp == P_EPI) {
        // ---------------- weights by TMA, one MMA per rank ----------------
        if (lane == 0) {
            auto load_w = [&](int l) {  // [W_k^(l); W_p^(l)] into buffer l % 2
                const int bi = l & 1;
                uint8_t *dst = sm + LY::W + bi * LY::WBUF;
                mbar_expect_tx(&wbar[bi], LY::WBUF);
                for (int blk = 0; blk < D / 64; ++blk) {
                    tma_load_4d(dst + blk * LY::W_BLK, &mk, blk * 64, 0, l, h, &wbar[bi]);
                    tma_load_4d(dst + blk * LY::W_BLK + D * 128, &mp, blk * 64, 0, l, h, &wbar[bi]);
                }
            };
            int issued = 0;
            if (!p.stall)
                for (; issued < L && issued < 2; ++issued) load_w(issued);
            bool ok = mbar_wait(&a_ready, 0, status, lim);
            const uint32_t id = idesc_bf16(128, 2 * D, 0, 0);
            auto oa = [](int ks) { return (uint64_t)koff_k_sw128(ks, LY::A_BLK); };
            auto ow = [](int ks) { return (uint64_t)koff_k_sw128(ks, LY::W_BLK); };
            const uint64_t dA = make_desc(sb + LY::A, 16, 1024, 2);
            const uint64_t dAl = make_desc(sb + LY::A_LO, 16, 1024, 2);
            for (int l = 0; l < L && ok; ++l) {
                const int bi = l & 1;
                if (!mbar_wait(&wbar[bi], (l >> 1) & 1, status, lim)) { ok = false; break; }
                // the epilogue of rank l - 2 has read this accumulator
                if (l >= 2 && !mbar_wait(&tfree[bi], ((l - 2) >> 1) & 1, status, lim)) { ok = false; break; }
                fence_after_sync();
                const uint64_t dW = make_desc(sb + LY::W + bi * LY::WBUF, 16, 1024, 2);
                // the anchor as a bf16 hi / lo pair: (a_hi + a_lo) W^T, the weights exact bf16
                mma_steps<D / 16>(tb + bi * 2 * D, id, dA, dW, oa, ow, false);
                mma_steps<D / 16>(tb + bi * 2 * D, id, dAl, dW, oa, ow, true);
                mma_commit(&full[bi]);
                if (issued < L) {  // W of rank l + 2 into this buffer once the MMA has read it
                    if (!mbar_wait(&full[bi], (l >> 1) & 1, status, lim)) { ok = false; break; }
                    load_w(issued++);
                }
            }
            if (!ok) failed_sh = 1;
            mma_commit(&drain);
            mbar_wait(&drain, 0, nullptr, lim);
            // after a failure, weight loads still in flight land before the CTA exits
            if (!ok)
                for (int l = issued > 2 ? issued - 2 : 0; l < issued; ++l)
                    mbar_wait(&wbar[l & 1], (l >> 1) & 1, nullptr, kStallTestPolls);
        }
    } else {
        // ---------------- anchor, then the residual chain, rank by rank ----------------
        const int q = warp & 3, hs = warp >> 2;  // TMEM lane quarter, column half
        const int row = 32 * q + lane, t = t0 + row;
        const bool live = t < T;
        const int c_base = hs * HALF;
        const size_t tok = ((size_t)b * T + t) * H + h;
        const __nv_bfloat16 *x = (const __nv_bfloat16 *)p.x;
        const __nv_bfloat16 *v = (const __nv_bfloat16 *)p.v;
        float r[HALF];
#pragma unroll
        for (int c8 = 0; c8 < HALF; c8 += 8) {
            const int col = c_base + c8;
            float a8[8], xf[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) a8[i] = 0.f;
            if (live) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (t - j >= 0) {
                        const uint4 xv = *reinterpret_cast<const uint4 *>(x + (((size_t)b * T + t - j) * H + h) * D + col);
                        unpack8(xv, xf);
                        const float *cj = p.conv + ((size_t)h * 4 + j) * D + col;
                        const float4 c0 = *reinterpret_cast<const float4 *>(cj);
                        const float4 c1 = *reinterpret_cast<const float4 *>(cj + 4);
                        const float cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                        for (int i = 0; i < 8; ++i) a8[i] = fmaf(cw[i], xf[i], a8[i]);
                    }
                }
                unpack8(*reinterpret_cast<const uint4 *>(v + tok * D + col), r + c8);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) r[c8 + i] = 0.f;
            }
            uint4 hi, lo;
            split8(a8, hi, lo);
            const uint32_t off = sw128_off(row, col, LY::A_BLK);
            st16(sm + LY::A, off, hi);
            st16(sm + LY::A_LO, off, lo);
        }
        fence_async_smem();
        fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_ready);

        __nv_bfloat16 *uo = (__nv_bfloat16 *)p.u, *wo = (__nv_bfloat16 *)p.w;
        bool ok = true;
        for (int l = 0; l < L && ok; ++l) {
            const int bi = l & 1;
            if (!mbar_wait(&full[bi], (l >> 1) & 1, status, lim)) { ok = false; break; }
            fence_after_sync();
            const float bl = live ? p.beta[tok * L + l] : 0.f;
            const size_t orow = (tok * L + l) * D;
            // 16 columns at a time (directions, then gains), few registers beyond the residual
#pragma unroll
            for (int ci = 0; ci < HALF / 16; ++ci) {
                const int col = c_base + 16 * ci;
                float kk[16];
                tmem_ld16(taddr(tb, 32 * q, bi * 2 * D + col), kk);
                tmem_wait_ld();
                if (live) {
                    *reinterpret_cast<uint4 *>(wo + orow + col) = pack8(kk);
                    *reinterpret_cast<uint4 *>(wo + orow + col + 8) = pack8(kk + 8);
                }
                float pp[16];
                tmem_ld16(taddr(tb, 32 * q, bi * 2 * D + D + col), pp);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float z = pp[j] * r[16 * ci + j];
                    const float dl = 0.5f * z * (1.f + erff(z * kRsqrt2));
                    r[16 * ci + j] -= dl;
                    pp[j] = bl * dl;
                }
                if (live) {
                    *reinterpret_cast<uint4 *>(uo + orow + col) = pack8(pp);
                    *reinterpret_cast<uint4 *>(uo + orow + col + 8) = pack8(pp + 8);
                }
            }
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tfree[bi]);
        }
        if (!ok) failed_sh = 1;
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == P_EPI) tmem_dealloc(tb, LY::TCOLS);
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
bool weight_map(CUtensorMap *m, const void *base, int H, int L, int d) {
    auto enc = map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)d, (cuuint64_t)L, (cuuint64_t)H};
    const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)d * d * 2, (cuuint64_t)L * d * d * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)d, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_producer_t(const ProducerArgs &a, cudaStream_t s) {
    CUtensorMap mk, mp;
    if (!weight_map(&mk, a.Wk, a.H, a.L, D) || !weight_map(&mp, a.Wp, a.H, a.L, D))
        return cudaErrorInvalidValue;
    using LY = ProdLayout<D>;
    auto kern = write_producer_kernel<D>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)LY::BYTES);
    if (err != cudaSuccess) return err;
    dim3 grid((a.T + PT - 1) / PT, a.H, a.B);
    launch_probe_mark(s);
    kern<<<grid, P_THREADS, LY::BYTES, s>>>(a, mk, mp);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_write_producer(const ProducerArgs &a, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    return a.d == 128 ? launch_producer_t<128>(a, s) : launch_producer_t<64>(a, s);
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
