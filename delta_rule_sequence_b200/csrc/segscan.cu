// segscan.cu -- the segmented inter-chunk scan, for few sequences that are long.
//
// When B*H is too small for one in-order pass per (sequence, value slice) to fill the GPU, each
// sequence is cut into G segments of T/G tokens and the segments are processed in parallel
// ("Sequential Parallel Duality in Prefix Scannable Models", method overview and key design 2:
// every chunk -- here every segment -- is encoded as an affine element (E, f) with S -> S E + f,
// the elements are combined by a static Blelloch scan, and each chunk is then run from its
// exclusive prefix state):
//   1. encode: the ordinary scan over the segment view [B*G, T/G, H, d] (no copy: [B, T, ...] is
//      [B, G, T/G, ...]) twice, without outputs: from S0 = I with the write switched off, which
//      leaves E_g in S_final, and from S0 = 0 with the write, which leaves f_g;
//   2. Blelloch over the G elements of each (b, h): the up-sweep composes sibling elements
//      (x then y: (E_x E_y, f_x E_y + f_y)); the down-sweep carries states instead of elements
//      -- a node's state goes to its left child unchanged and to its right child as
//      state E_left + f_left -- so each leaf receives S0 followed by every segment before it;
//   3. the ordinary scan over the segment view from those entry states, with outputs; the exit
//      state is the last leaf's state advanced over its own segment.
// Steps 1 and 3 reuse the route's kernels (and, on the Gated-DeltaNet route, one shared set of
// per-chunk records).  Step 2 is fp32 on CUDA cores: G <= 16, and each composition is a
// (rows x d) by (d x d) product.

#include "common.cuh"

namespace prism {

cudaError_t launch_scan_simt(const ScanArgs &a, bool io_f32, cudaStream_t s);
cudaError_t launch_gdn_prep(const ScanArgs &a, void *ws, cudaStream_t s);
cudaError_t launch_gdn_state(const ScanArgs &a, const void *ws, cudaStream_t s);
cudaError_t launch_lrank_prep(const ScanArgs &a, void *ws, cudaStream_t s);
cudaError_t launch_lrank_state(const ScanArgs &a, const void *ws, cudaStream_t s);

namespace {

constexpr int RB = 16;     // rows per CTA of a (rows x d) x (d x d) product
constexpr int NTH = 256;

// Row block `rb` of out = x E (+ add): rows rb*RB .. rb*RB+RB-1 of x (nrows x D), E (D x D)
// staged in shared memory.
// x and out may be the same array (prism_state_fold in place), so neither is restrict-qualified.
template <int D>
__device__ __forceinline__ void rows_times(const float *x, const float *__restrict__ E,
                                           const float *__restrict__ add, float *out,
                                           int nrows, int rb, float *sE, float *sx) {
    for (int e = threadIdx.x; e < D * D / 4; e += NTH)
        reinterpret_cast<float4 *>(sE)[e] = reinterpret_cast<const float4 *>(E)[e];
    const int r0 = rb * RB;
    for (int e = threadIdx.x; e < RB * D; e += NTH) {
        const int r = e / D, c = e % D;
        sx[r * (D + 1) + c] = (r0 + r < nrows) ? x[(size_t)(r0 + r) * D + c] : 0.f;
    }
    __syncthreads();
    constexpr int TPR = NTH / RB;      // threads per row
    constexpr int CPT = D / TPR;       // columns per thread
    const int r = threadIdx.x / TPR, c0 = (threadIdx.x % TPR) * CPT;
    float acc[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) acc[j] = 0.f;
#pragma unroll 4
    for (int k = 0; k < D; ++k) {
        const float xv = sx[r * (D + 1) + k];
#pragma unroll
        for (int j = 0; j < CPT; ++j) acc[j] = fmaf(xv, sE[k * D + c0 + j], acc[j]);
    }
    if (r0 + r < nrows) {
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            const size_t idx = (size_t)(r0 + r) * D + c0 + j;
            out[idx] = acc[j] + (add ? add[idx] : 0.f);
        }
    }
}

// Segment elements of head (b, h): leaf g at Eleaf/Fleaf index (b G + g) H + h; internal node
// (level l >= 1, position i) at Eint/Fint index (b H + h)(G - 1) + (G - G / 2^(l-1)) + i.
struct SegTree {
    const float *Eleaf, *Fleaf;
    float *Eint, *Fint;
    float *Sent;       // entry states, [B G, H, dv, dk]: slot g of head (b, h) at (b G + g) H + h
    int B, H, G, dk, dv;
};

__device__ __forceinline__ size_t leaf_idx(const SegTree &t, int b, int h, int g) {
    return ((size_t)b * t.G + g) * t.H + h;
}
__device__ __forceinline__ size_t int_idx(const SegTree &t, int b, int h, int level, int i) {
    return ((size_t)b * t.H + h) * (t.G - 1) + (t.G - (t.G >> (level - 1))) + i;
}
template <int D>
__device__ __forceinline__ const float *node_E(const SegTree &t, int b, int h, int lv, int pos) {
    return lv == 0 ? t.Eleaf + leaf_idx(t, b, h, pos) * D * D : t.Eint + int_idx(t, b, h, lv, pos) * D * D;
}
template <int D>
__device__ __forceinline__ const float *node_F(const SegTree &t, int b, int h, int lv, int pos) {
    const size_t fe = (size_t)t.dv * D;
    return lv == 0 ? t.Fleaf + leaf_idx(t, b, h, pos) * fe : t.Fint + int_idx(t, b, h, lv, pos) * fe;
}

// Up-sweep, level `level` (>= 1): node(level, i) = node(level-1, 2i) (+) node(level-1, 2i+1),
// i.e. E = E_x E_y (row blocks 0 .. D/RB-1) and f = f_x E_y + f_y (the row blocks after those).
// grid: x = row blocks over the D + dv rows, y = node i, z = b * H + h.
template <int D>
__global__ void __launch_bounds__(NTH) seg_compose_kernel(SegTree t, int level) {
    extern __shared__ float smem[];
    float *sE = smem, *sx = smem + D * D;
    const int i = blockIdx.y, b = blockIdx.z / t.H, h = blockIdx.z % t.H;
    const float *Ex = node_E<D>(t, b, h, level - 1, 2 * i), *Fx = node_F<D>(t, b, h, level - 1, 2 * i);
    const float *Ey = node_E<D>(t, b, h, level - 1, 2 * i + 1), *Fy = node_F<D>(t, b, h, level - 1, 2 * i + 1);
    float *Eo = t.Eint + int_idx(t, b, h, level, i) * D * D;
    float *Fo = t.Fint + int_idx(t, b, h, level, i) * (size_t)t.dv * D;
    constexpr int eblocks = (D + RB - 1) / RB;
    if ((int)blockIdx.x < eblocks)
        rows_times<D>(Ex, Ey, nullptr, Eo, D, blockIdx.x, sE, sx);
    else
        rows_times<D>(Fx, Ey, Fy, Fo, t.dv, blockIdx.x - eblocks, sE, sx);
}

// Down-sweep, level `level` (>= 1): the state of node(level, i) sits in slot i 2^level; its right
// child's slot i 2^level + 2^(level-1) receives state E(left) + f(left), left = node(level-1, 2i).
// grid: x = row blocks over dv rows, y = node i, z = b * H + h.
template <int D>
__global__ void __launch_bounds__(NTH) seg_apply_kernel(SegTree t, int level) {
    extern __shared__ float smem[];
    float *sE = smem, *sx = smem + D * D;
    const int i = blockIdx.y, b = blockIdx.z / t.H, h = blockIdx.z % t.H;
    const size_t fe = (size_t)t.dv * D;
    const int src = i << level, dst = src + (1 << (level - 1));
    rows_times<D>(t.Sent + leaf_idx(t, b, h, src) * fe, node_E<D>(t, b, h, level - 1, 2 * i),
                  node_F<D>(t, b, h, level - 1, 2 * i), t.Sent + leaf_idx(t, b, h, dst) * fe, t.dv,
                  blockIdx.x, sE, sx);
}

// Slot 0 of every head <- S0 (or zeros).  grid: x = blocks of 1024 floats, z = b * H + h.
__global__ void __launch_bounds__(NTH) seg_init_kernel(SegTree t, const float *S0) {
    const int b = blockIdx.z / t.H, h = blockIdx.z % t.H;
    const size_t fe = (size_t)t.dv * t.dk;
    float *O = t.Sent + leaf_idx(t, b, h, 0) * fe;
    const float *I = S0 ? S0 + ((size_t)b * t.H + h) * fe : nullptr;
    for (size_t idx = (size_t)blockIdx.x * 1024 + threadIdx.x; idx < fe && idx < (size_t)(blockIdx.x + 1) * 1024;
         idx += NTH)
        O[idx] = I ? I[idx] : 0.f;
}

// Exit state S_final = Sent[G-1] E_{G-1} + f_{G-1}.  grid: x = row blocks over dv, z = b * H + h.
template <int D>
__global__ void __launch_bounds__(NTH) seg_exit_kernel(SegTree t, float *S_final) {
    extern __shared__ float smem[];
    float *sE = smem, *sx = smem + D * D;
    const int b = blockIdx.z / t.H, h = blockIdx.z % t.H, g = t.G - 1;
    const size_t fe = (size_t)t.dv * D;
    rows_times<D>(t.Sent + leaf_idx(t, b, h, g) * fe, t.Eleaf + leaf_idx(t, b, h, g) * D * D,
                  t.Fleaf + leaf_idx(t, b, h, g) * fe, S_final + ((size_t)b * t.H + h) * fe, t.dv,
                  blockIdx.x, sE, sx);
}

template <int D>
cudaError_t combine(const SegTree &t, const float *S0, float *S_final, cudaStream_t s) {
    const size_t smem = ((size_t)D * D + (size_t)RB * (D + 1)) * sizeof(float);
    cudaError_t err = cudaFuncSetAttribute(seg_compose_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(seg_apply_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(seg_exit_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const int BH = t.B * t.H;
    const int vblocks = (t.dv + RB - 1) / RB, eblocks = (D + RB - 1) / RB;
    int levels = 0;
    while ((1 << levels) < t.G) ++levels;
    const int iblocks = (int)(((size_t)t.dv * t.dk + 1023) / 1024);
    launch_probe_mark(s);
    seg_init_kernel<<<dim3(iblocks, 1, BH), NTH, 0, s>>>(t, S0);
    for (int lv = 1; lv < levels; ++lv) {  // up-sweep (the root's element is not needed)
        launch_probe_mark(s);
        seg_compose_kernel<D><<<dim3(eblocks + vblocks, t.G >> lv, BH), NTH, smem, s>>>(t, lv);
    }
    for (int lv = levels; lv >= 1; --lv) {  // down-sweep, root to leaves
        launch_probe_mark(s);
        seg_apply_kernel<D><<<dim3(vblocks, t.G >> lv, BH), NTH, smem, s>>>(t, lv);
    }
    if (S_final) {
        launch_probe_mark(s);
        seg_exit_kernel<D><<<dim3(vblocks, 1, BH), NTH, smem, s>>>(t, S_final);
    }
    return cudaGetLastError();
}

// S_final of a pass over no tokens: the entry state (S0, zero, or the identity under kS0Identity).
__global__ void __launch_bounds__(NTH) state_init_kernel(ScanArgs a, size_t n) {
    const size_t i = (size_t)blockIdx.x * NTH + threadIdx.x;
    if (i >= n) return;
    const int c = (int)(i % a.dk), r = (int)((i / a.dk) % a.dv);
    a.S_final[i] = (a.flags & kS0Identity) ? (r == c ? 1.f : 0.f) : (a.S0 ? a.S0[i] : 0.f);
}

// S_out = S_in E + f for every (b, h): S_in, f, S_out [BH, dv, D], E [BH, D, D].  S_out may be
// S_in (each CTA stages its own rows before writing them).  grid: x = b * H + h, y = row blocks.
template <int D>
__global__ void __launch_bounds__(NTH) state_fold_kernel(const float *S_in, const float *E, const float *f,
                                                         float *S_out, int dv) {
    extern __shared__ float smem[];
    float *sE = smem, *sx = smem + D * D;
    const size_t bh = blockIdx.x, fe = (size_t)dv * D;
    rows_times<D>(S_in + bh * fe, E + bh * D * D, f + bh * fe, S_out + bh * fe, dv, blockIdx.y, sE, sx);
}

template <int D>
cudaError_t fold_t(int BH, int dv, const float *S_in, const float *E, const float *f, float *S_out,
                   cudaStream_t s) {
    const size_t smem = ((size_t)D * D + (size_t)RB * (D + 1)) * sizeof(float);
    cudaError_t err = cudaFuncSetAttribute(state_fold_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    launch_probe_mark(s);
    state_fold_kernel<D><<<dim3(BH, (dv + RB - 1) / RB), NTH, smem, s>>>(S_in, E, f, S_out, dv);
    return cudaGetLastError();
}

}  // namespace

// A scan pass over T = 0 tokens: S_final receives the entry state (nothing if S_final is NULL).
cudaError_t launch_state_init(const ScanArgs &a, cudaStream_t s) {
    const size_t n = (size_t)a.B * a.H * a.dv * a.dk;
    if (!a.S_final || n == 0) return cudaSuccess;
    launch_probe_mark(s);
    state_init_kernel<<<(unsigned)((n + NTH - 1) / NTH), NTH, 0, s>>>(a, n);
    return cudaGetLastError();
}

// S_out = S_in E + f per (b, h) (S_in NULL: S_out = f).  dk in {32, 64, 128}.
cudaError_t launch_state_fold(int BH, int dk, int dv, const float *S_in, const float *E, const float *f,
                              float *S_out, cudaStream_t s) {
    if (BH == 0) return cudaSuccess;
    if (!S_in) {
        launch_probe_mark(s);
        return cudaMemcpyAsync(S_out, f, (size_t)BH * dv * dk * sizeof(float), cudaMemcpyDeviceToDevice, s);
    }
    switch (dk) {
        case 128: return fold_t<128>(BH, dv, S_in, E, f, S_out, s);
        case 64: return fold_t<64>(BH, dv, S_in, E, f, S_out, s);
        case 32: return fold_t<32>(BH, dv, S_in, E, f, S_out, s);
    }
    return cudaErrorInvalidValue;
}

// The affine map of each (b, h) sequence of `a` (dk == dv): E into e_out ([B, H, dk, dk]) from
// S0 = I with the write off, f into f_out ([B, H, dv, dk]) from S0 = 0 with the write; no outputs.
cudaError_t launch_segment_element(const ScanArgs &a, int route, bool io_f32, void *ws, float *e_out,
                                   float *f_out, cudaStream_t s) {
    auto pass = [&](const ScanArgs &x) -> cudaError_t {
        switch (route) {
            case 3: return launch_lrank_state(x, ws, s);
            case 2: return launch_gdn_state(x, ws, s);
            default: return launch_scan_simt(x, io_f32, s);
        }
    };
    cudaError_t err = cudaSuccess;
    if (route == 2 && a.T > 0 && (err = launch_gdn_prep(a, ws, s)) != cudaSuccess) return err;
    if (route == 3 && a.T > 0 && (err = launch_lrank_prep(a, ws, s)) != cudaSuccess) return err;
    ScanArgs e = a;
    e.S0 = nullptr;
    e.o = nullptr;
    e.flags = (a.flags & (kForceWkLo | kStallTest | kStallPrep)) | kNoWrite | kS0Identity | kNoOutput;
    e.S_final = e_out;
    if ((err = a.T == 0 ? launch_state_init(e, s) : pass(e)) != cudaSuccess) return err;
    ScanArgs f = a;
    f.S0 = nullptr;
    f.o = nullptr;
    f.flags = (a.flags & (kForceWkLo | kStallTest | kStallPrep)) | kNoOutput;
    f.S_final = f_out;
    return a.T == 0 ? launch_state_init(f, s) : pass(f);
}

// Kernels one segmented scan launches besides the passes: slot-0 init, the up- and down-sweep
// levels, and the exit state.
int segmented_combine_launches(int G, bool with_state) {
    int levels = 0;
    while ((1 << levels) < G) ++levels;
    return 1 + (levels > 0 ? levels - 1 : 0) + levels + (with_state ? 1 : 0);
}

// Workspace of the segmented scan after the status block (and, on the Gated-DeltaNet route, the
// per-chunk records of the segment view): leaf elements, internal nodes, entry states.
size_t segmented_extra_bytes(int B, int H, int G, int dk, int dv) {
    const size_t ee = (size_t)dk * dk * 4, fe = (size_t)dv * dk * 4;
    return (size_t)B * G * H * (ee + fe) + (size_t)B * H * (G - 1) * (ee + fe) + (size_t)B * G * H * fe;
}

// route: 0 fp32 CUDA cores, 2 Gated-DeltaNet prep + state kernels, 3 rank-L prep + state kernels.
// ws: the caller's workspace (status word first); `rec_bytes` bytes of records follow the status
// block on route 2, and the segment arrays follow those.
cudaError_t launch_segmented(const ScanArgs &a, int route, bool io_f32, int G, void *ws,
                             size_t rec_bytes, cudaStream_t s) {
    const int Ts = a.T / G;
    ScanArgs v = a;  // the segment view [B*G, T/G, H, ...]
    v.B = a.B * G;
    v.T = Ts;
    v.S0 = nullptr;
    uint8_t *base = (uint8_t *)ws + rec_bytes;
    const size_t ee = (size_t)a.dk * a.dk, fe = (size_t)a.dv * a.dk;
    SegTree t;
    t.B = a.B; t.H = a.H; t.G = G; t.dk = a.dk; t.dv = a.dv;
    float *Eleaf = (float *)base;
    float *Fleaf = Eleaf + (size_t)a.B * G * a.H * ee;
    float *Eint = Fleaf + (size_t)a.B * G * a.H * fe;
    float *Fint = Eint + (size_t)a.B * a.H * (G - 1) * ee;
    float *Sent = Fint + (size_t)a.B * a.H * (G - 1) * fe;
    t.Eleaf = Eleaf; t.Fleaf = Fleaf; t.Eint = Eint; t.Fint = Fint; t.Sent = Sent;

    auto pass = [&](const ScanArgs &x) -> cudaError_t {
        switch (route) {
            case 3: return launch_lrank_state(x, ws, s);
            case 2: return launch_gdn_state(x, ws, s);
            default: return launch_scan_simt(x, io_f32, s);
        }
    };
    cudaError_t err = cudaSuccess;
    if (route == 2 && (err = launch_gdn_prep(v, ws, s)) != cudaSuccess) return err;
    if (route == 3 && (err = launch_lrank_prep(v, ws, s)) != cudaSuccess) return err;
    // 1. encode: E_g (identity rows, no write) and f_g (zero state, with the write)
    ScanArgs e = v;
    e.flags = (a.flags & (kForceWkLo | kStallTest | kStallPrep)) | kNoWrite | kS0Identity | kNoOutput;
    e.S_final = Eleaf;
    if ((err = pass(e)) != cudaSuccess) return err;
    ScanArgs f = v;
    f.flags = (a.flags & (kForceWkLo | kStallTest | kStallPrep)) | kNoOutput;
    f.S_final = Fleaf;
    if ((err = pass(f)) != cudaSuccess) return err;
    // 2. Blelloch over the segment elements -> entry states; exit state
    err = a.dk == 128 ? combine<128>(t, a.S0, a.S_final, s)
        : a.dk == 64  ? combine<64>(t, a.S0, a.S_final, s)
                      : combine<32>(t, a.S0, a.S_final, s);
    if (err != cudaSuccess) return err;
    // 3. every segment from its entry state, with outputs
    ScanArgs r = v;
    r.S0 = Sent;
    r.S_final = nullptr;
    return pass(r);
}

}  // namespace prism
