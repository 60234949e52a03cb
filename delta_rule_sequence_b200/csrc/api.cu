// api.cu -- the C ABI of libprism.so (declared in include/prism.h): argument validation, plan
// selection and kernel launches.  No allocation, no synchronisation except in
// prism_query_device_status, no printing.

#include <stdint.h>

#include "common.cuh"
#include "producer.cuh"

namespace prism {
cudaError_t launch_scan_simt(const ScanArgs &a, bool io_f32, cudaStream_t s);
cudaError_t launch_decode(const ScanArgs &a, bool io_f32, cudaStream_t s);
cudaError_t decode_status(uint32_t *out);
cudaError_t launch_state_init(const ScanArgs &a, cudaStream_t s);
size_t gdn_workspace_bytes(int B, int H, int T, int dk);
cudaError_t launch_scan_gdn(const ScanArgs &a, void *ws, cudaStream_t s);
size_t lrank_workspace_bytes(int B, int H, int T, int dk);
cudaError_t launch_scan_lrank(const ScanArgs &a, void *ws, cudaStream_t s);
int segmented_combine_launches(int G, bool with_state);
size_t segmented_extra_bytes(int B, int H, int G, int dk, int dv);
cudaError_t launch_segmented(const ScanArgs &a, int route, bool io_f32, int G, void *ws,
                             size_t rec_bytes, cudaStream_t s);
cudaError_t launch_segment_element(const ScanArgs &a, int route, bool io_f32, void *ws, float *e_out,
                                   float *f_out, cudaStream_t s);
cudaError_t launch_state_fold(int BH, int dk, int dv, const float *S_in, const float *E, const float *f,
                              float *S_out, cudaStream_t s);
cudaError_t noalloc_status(uint32_t *out);
size_t bwd_workspace_bytes(int B, int H, int T, int dk, int dv, bool io_f32);
cudaError_t launch_scan_bwd(const ScanArgs &f, const void *dO, const float *dS_final, float *dq,
                            float *dk, float *dv, float *dalpha, float *dbeta, float *du, float *dw,
                            float *dS0, void *ws, bool io_f32, cudaStream_t s);
}  // namespace prism

namespace {

int g_debug_flags = 0;

// Armed launch probe of this host thread: the events to record before each launch of the next
// prism_scan_fwd / prism_step_decode call, and after its last launch.
constexpr int kMaxProbeEvents = 64;
struct LaunchProbe {
    void *events[kMaxProbeEvents] = {};  // copied from the caller: its array need not outlive the arming call
    int n = 0, next = 0;
};
thread_local LaunchProbe t_probe;

// The CUDA error behind this thread's last PRISM_ERR_CUDA (cudaSuccess if none yet).
thread_local cudaError_t t_last_cuda_error = cudaSuccess;

prism_status cuda_status(cudaError_t err) {
    if (err == cudaSuccess) return PRISM_OK;
    t_last_cuda_error = err;
    return PRISM_ERR_CUDA;
}

// Records the probe's last event after a probed call's final launch and disarms the probe.
void probe_finish(cudaStream_t s) {
    prism::launch_probe_mark(s);
    t_probe = LaunchProbe{};
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
bool width_ok(int d) { return d == 32 || d == 64 || d == 128; }

// Shared checks of prism_scan_fwd and prism_step_decode.
prism_status check_common(const prism_shape *s, const void *q, const void *k, const void *v,
                          const float *alpha, const float *beta, const void *u, const void *w) {
    if (!s) return PRISM_ERR_INVALID_ARG;
    if (s->B < 0 || s->H < 0 || s->T < 0) return PRISM_ERR_INVALID_ARG;
    if (s->io != PRISM_BF16 && s->io != PRISM_F32) return PRISM_ERR_INVALID_ARG;
    if (s->L < 1) return PRISM_ERR_INVALID_ARG;  // L = 0 would have no write at all
    if (s->dk < 1 || s->dv < 1) return PRISM_ERR_INVALID_ARG;
    if (!width_ok(s->dk) || !width_ok(s->dv) || s->L > 8) return PRISM_ERR_UNSUPPORTED;
    if (s->B > 65535 || s->H > 65535) return PRISM_ERR_UNSUPPORTED;
    // With no tokens nothing below is read (an empty tensor may even have a NULL data pointer).
    const bool work = (long long)s->B * s->H * s->T > 0;
    if (!work) return PRISM_OK;
    if ((u == nullptr) != (w == nullptr)) return PRISM_ERR_INVALID_ARG;
    if (u == nullptr && s->L != 1) return PRISM_ERR_INVALID_ARG;
    if (!q || !k || !alpha || !beta) return PRISM_ERR_INVALID_ARG;
    if (u == nullptr && v == nullptr) return PRISM_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, u, w};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return PRISM_ERR_INVALID_ARG;
    if (((uintptr_t)alpha & 3u) || ((uintptr_t)beta & 3u)) return PRISM_ERR_INVALID_ARG;
    return PRISM_OK;
}

// Which kernels a prism_scan_fwd call with this shape runs: nothing but the exit state when there
// are no tokens; the two-kernel tensor-core schedule (per-chunk prep, then the in-order state
// kernel) for the Gated-DeltaNet or the rank-L write; the fp32 CUDA-core kernel otherwise.
enum class Plan { Empty, Simt, TcGdnSplit, TcRankLSplit };

Plan plan_for(const prism_shape *s, bool gdn_write) {
    if (s->T <= 0) return Plan::Empty;
    const bool tc = s->io == PRISM_BF16 && s->dk == s->dv && (s->dk == 64 || s->dk == 128);
    if (!tc) return Plan::Simt;
    return gdn_write ? Plan::TcGdnSplit : Plan::TcRankLSplit;
}

bool split_plan(Plan p) { return p == Plan::TcGdnSplit || p == Plan::TcRankLSplit; }

// Route number of the segmented scan and the segment element: 0 fp32, 2 GDN split, 3 rank-L split.
int route_of(Plan p) {
    switch (p) {
        case Plan::TcGdnSplit: return 2;
        case Plan::TcRankLSplit: return 3;
        default: return 0;
    }
}

// Debug flag bits (prism_debug_set_flags): 2 = take the segmented scan whenever the shape allows
// it, 4 = never take it, 8 = the stall test of the Gated-DeltaNet state kernel (its waits give up),
// 16 = the state kernel's Wk_lo term from the first chunk on, whatever the size of the state,
// 32 = the stall test of the per-chunk prep kernels, 64 = of the write producer, 128 = of the
// bulk-copy decode kernel.
constexpr int kForceSegments = 2, kNoSegments = 4, kDebugStall = 8, kDebugForceWkLo = 16,
              kDebugStallPrep = 32, kDebugStallProducer = 64, kDebugStallDecode = 128;

// Number of segments G of the segmented inter-chunk scan (1 = one in-order pass per sequence).
// It needs dk == dv (the identity pass) and T divisible by G with at least one chunk per segment.
int sm_count() {
    static int sms[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        sms[dev] = n;
    }
    return sms[dev];
}

// Measured on B200: on the Gated-DeltaNet route (whose in-order pass is latency-bound per chunk),
// cutting 16 sequence slices of 65536 tokens into 16 segments halves the time; on the fused rank-L
// route (one CTA per SM) the tripled work of the segmented scan does not pay.  So segments are
// taken on the Gated-DeltaNet route when the in-order passes fill at most a quarter of the SMs.
int segments_for(const prism_shape *s, bool gdn_write) {
    if ((g_debug_flags & kNoSegments) || s->dk != s->dv || s->T < 128) return 1;
    auto largest_G = [&](int max_g, int min_len) {
        for (int G = 16; G >= 2; G /= 2)
            if (G <= max_g && s->T % G == 0 && s->T / G >= min_len) return G;
        return 1;
    };
    if (g_debug_flags & kForceSegments) return largest_G(16, 64);
    if (!split_plan(plan_for(s, gdn_write))) return 1;
    const long long chains = (long long)s->B * s->H * (s->dv == 128 ? 4 : 1);
    const int sms = sm_count();
    if (chains * 4 > sms || s->T < 4096) return 1;
    return largest_G((int)(sms / chains), 256);
}

size_t records_bytes(const prism_shape *s, Plan plan, int G) {
    if (!split_plan(plan) || s->T <= 0 || s->B == 0 || s->H == 0) return prism::kStatusBytes;
    return plan == Plan::TcGdnSplit ? prism::gdn_workspace_bytes(s->B * G, s->H, s->T / G, s->dk)
                                    : prism::lrank_workspace_bytes(s->B * G, s->H, s->T / G, s->dk);
}

prism::ScanArgs make_args(const prism_shape *s, const void *q, const void *k, const void *v,
                          const float *alpha, const float *beta, const void *u, const void *w,
                          const float *S0, void *o, float *S_final, uint32_t *status) {
    prism::ScanArgs a;
    a.B = s->B; a.H = s->H; a.T = s->T; a.dk = s->dk; a.dv = s->dv; a.L = s->L;
    a.chunk = s->chunk;
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta; a.u = u; a.w = w;
    a.S0 = S0; a.o = o; a.S_final = S_final; a.status = status;
    a.flags = 0;
    return a;
}

}  // namespace

namespace prism {
// Every check of a prism_scan_fwd call that does not involve the workspace (prism_scan_fwd_noalloc
// runs these before it sizes anything).
prism_status check_scan_call(const prism_shape *shape, const void *q, const void *k, const void *v,
                             const float *alpha, const float *beta, const void *u, const void *w,
                             const float *S0, const void *o, const float *S_final) {
    prism_status st = check_common(shape, q, k, v, alpha, beta, u, w);
    if (st != PRISM_OK) return st;
    if (shape->chunk != 64 && shape->chunk != 128) return PRISM_ERR_INVALID_ARG;
    if ((S0 && !aligned16(S0)) || (S_final && !aligned16(S_final))) return PRISM_ERR_INVALID_ARG;
    const long long work = (long long)shape->B * shape->H * shape->T;
    if (work > 0 && (!o || !aligned16(o))) return PRISM_ERR_INVALID_ARG;
    if (o && (o == q || o == k || o == v || o == u || o == w)) return PRISM_ERR_INVALID_ARG;
    return PRISM_OK;
}

void launch_probe_mark(cudaStream_t s) {
    LaunchProbe &p = t_probe;
    if (p.next < p.n) cudaEventRecord((cudaEvent_t)p.events[p.next++], s);
}
}  // namespace prism

extern "C" {

// The workspace and launch count cover the larger of the two write forms (Gated-DeltaNet write
// when u, w are NULL, rank-L otherwise), since the shape alone does not say which one is used.
prism_status prism_scan_fwd_workspace_size(const prism_shape *shape, size_t *bytes) {
    if (!shape || !bytes) return PRISM_ERR_INVALID_ARG;
    size_t need = 0;
    for (int gdn = 0; gdn < 2; ++gdn) {
        if (gdn && shape->L != 1) continue;  // the Gated-DeltaNet write exists only for L = 1
        const Plan plan = plan_for(shape, gdn);
        const int G = segments_for(shape, gdn);
        size_t n = records_bytes(shape, plan, G);
        if (G > 1) n += prism::segmented_extra_bytes(shape->B, shape->H, G, shape->dk, shape->dv);
        if (n > need) need = n;
    }
    *bytes = need;
    return PRISM_OK;
}

prism_status prism_scan_fwd_launch_count(const prism_shape *shape, int *launches) {
    if (!shape || !launches) return PRISM_ERR_INVALID_ARG;
    int most = 0;
    for (int gdn = 0; gdn < 2; ++gdn) {
        if (gdn && shape->L != 1) continue;
        const Plan plan = plan_for(shape, gdn);
        const int G = segments_for(shape, gdn);
        const bool split = split_plan(plan);
        int n = split ? 2 : 1;
        if (G > 1) n = (split ? 1 : 0) + 3 + prism::segmented_combine_launches(G, true);
        if (n > most) most = n;
    }
    if (shape->B == 0 || shape->H == 0) most = 0;
    *launches = most;
    return PRISM_OK;
}

prism_status prism_scan_fwd(const prism_shape *shape, const void *q, const void *k,
                            const void *v, const float *alpha, const float *beta,
                            const void *u, const void *w, const float *S0, void *o,
                            float *S_final, void *workspace, size_t ws_bytes, void *stream) {
    prism_status st = prism::check_scan_call(shape, q, k, v, alpha, beta, u, w, S0, o, S_final);
    if (st != PRISM_OK) return st;
    size_t need = 0;
    prism_scan_fwd_workspace_size(shape, &need);
    if (!workspace || ws_bytes < need || ((uintptr_t)workspace & 255u)) return PRISM_ERR_INVALID_ARG;

    cudaStream_t s = (cudaStream_t)stream;
    uint32_t *status = (uint32_t *)workspace;
    if (shape->B == 0 || shape->H == 0) return PRISM_OK;
    if (shape->T == 0 && !S_final) return PRISM_OK;

    prism::ScanArgs a = make_args(shape, q, k, v, alpha, beta, u, w, S0, o, S_final, status);
    if (g_debug_flags & kDebugStall) a.flags |= prism::kStallTest;
    if (g_debug_flags & kDebugForceWkLo) a.flags |= prism::kForceWkLo;
    if (g_debug_flags & kDebugStallPrep) a.flags |= prism::kStallPrep;
    const bool io_f32 = shape->io == PRISM_F32;
    cudaError_t err;
    const Plan plan = plan_for(shape, u == nullptr);
    const int G = segments_for(shape, u == nullptr);
    if (G > 1) {
        err = prism::launch_segmented(a, route_of(plan), io_f32, G, workspace, records_bytes(shape, plan, G), s);
    } else {
        switch (plan) {
            case Plan::TcGdnSplit: err = prism::launch_scan_gdn(a, workspace, s); break;
            case Plan::TcRankLSplit: err = prism::launch_scan_lrank(a, workspace, s); break;
            case Plan::Empty: err = prism::launch_state_init(a, s); break;  // S_final = S0
            default: err = prism::launch_scan_simt(a, io_f32, s); break;
        }
    }
    probe_finish(s);
    return cuda_status(err);
}

prism_status prism_scan_segment_element(const prism_shape *shape, const void *q, const void *k,
                                        const void *v, const float *alpha, const float *beta,
                                        const void *u, const void *w, float *E, float *f,
                                        void *workspace, size_t ws_bytes, void *stream) {
    prism_status st = check_common(shape, q, k, v, alpha, beta, u, w);
    if (st != PRISM_OK) return st;
    if (shape->chunk != 64 && shape->chunk != 128) return PRISM_ERR_INVALID_ARG;
    if (shape->dk != shape->dv) return PRISM_ERR_UNSUPPORTED;
    size_t need = 0;
    prism_scan_fwd_workspace_size(shape, &need);
    if (!workspace || ws_bytes < need || ((uintptr_t)workspace & 255u)) return PRISM_ERR_INVALID_ARG;
    if (shape->B == 0 || shape->H == 0) return PRISM_OK;
    if (!E || !f || !aligned16(E) || !aligned16(f) || E == f) return PRISM_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    prism::ScanArgs a = make_args(shape, q, k, v, alpha, beta, u, w, nullptr, nullptr, nullptr,
                                  (uint32_t *)workspace);
    if (g_debug_flags & kDebugForceWkLo) a.flags |= prism::kForceWkLo;
    const Plan plan = plan_for(shape, u == nullptr);
    cudaError_t err = prism::launch_segment_element(a, route_of(plan), shape->io == PRISM_F32, workspace, E, f, s);
    probe_finish(s);
    return cuda_status(err);
}

prism_status prism_state_fold(int BH, int dk, int dv, const float *S_in, const float *E,
                              const float *f, float *S_out, void *stream) {
    if (BH < 0 || dk < 1 || dv < 1) return PRISM_ERR_INVALID_ARG;
    if (!width_ok(dk) || !width_ok(dv)) return PRISM_ERR_UNSUPPORTED;
    if (BH == 0) return PRISM_OK;
    if (!E || !f || !S_out || !aligned16(E) || !aligned16(f) || !aligned16(S_out) ||
        (S_in && !aligned16(S_in)))
        return PRISM_ERR_INVALID_ARG;
    if (S_out == E || S_out == f) return PRISM_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t err = prism::launch_state_fold(BH, dk, dv, S_in, E, f, S_out, s);
    probe_finish(s);
    return cuda_status(err);
}

prism_status prism_scan_bwd_workspace_size(const prism_shape *shape, size_t *bytes) {
    if (!shape || !bytes) return PRISM_ERR_INVALID_ARG;
    const prism_shape &s = *shape;
    if (s.B < 0 || s.H < 0 || s.T < 0 || !width_ok(s.dk) || !width_ok(s.dv)) return PRISM_ERR_INVALID_ARG;
    *bytes = prism::bwd_workspace_bytes(s.B, s.H, s.T, s.dk, s.dv, s.io == PRISM_F32);
    return PRISM_OK;
}

prism_status prism_scan_bwd(const prism_shape *shape, const void *q, const void *k, const void *v,
                            const float *alpha, const float *beta, const void *u, const void *w,
                            const float *S0, const void *dO, const float *dS_final, float *dq,
                            float *dk, float *dv, float *dalpha, float *dbeta, float *du, float *dw,
                            float *dS0, void *workspace, size_t ws_bytes, void *stream) {
    prism_status st = check_common(shape, q, k, v, alpha, beta, u, w);
    if (st != PRISM_OK) return st;
    if (shape->B == 0 || shape->H == 0) return PRISM_OK;
    size_t need = 0;
    prism_scan_bwd_workspace_size(shape, &need);
    if (!workspace || ws_bytes < need || ((uintptr_t)workspace & 255u)) return PRISM_ERR_INVALID_ARG;
    if ((S0 && !aligned16(S0)) || (dS_final && !aligned16(dS_final)) || (dS0 && !aligned16(dS0)))
        return PRISM_ERR_INVALID_ARG;
    const bool gdn = u == nullptr;
    if (shape->T > 0) {
        if (!dO || !aligned16(dO)) return PRISM_ERR_INVALID_ARG;
        for (const float *g : {dq, dk, dalpha, dbeta})
            if (!g || ((uintptr_t)g & 15u)) return PRISM_ERR_INVALID_ARG;
        if (gdn && (!dv || !aligned16(dv))) return PRISM_ERR_INVALID_ARG;
        if (!gdn && (!du || !dw || !aligned16(du) || !aligned16(dw))) return PRISM_ERR_INVALID_ARG;
        // no gradient may overlap another one or an input
        const void *outs[] = {dq, dk, gdn ? dv : nullptr, dalpha, dbeta, gdn ? nullptr : du,
                              gdn ? nullptr : dw, dS0};
        const void *ins[] = {q, k, v, alpha, beta, u, w, S0, dO, dS_final};
        for (int i = 0; i < 8; ++i) {
            if (!outs[i]) continue;
            for (int j = i + 1; j < 8; ++j)
                if (outs[i] == outs[j]) return PRISM_ERR_INVALID_ARG;
            for (const void *in : ins)
                if (in && in == outs[i]) return PRISM_ERR_INVALID_ARG;
        }
    }
    cudaStream_t s = (cudaStream_t)stream;
    prism::ScanArgs a = make_args(shape, q, k, v, alpha, beta, u, w, S0, nullptr, nullptr,
                                  (uint32_t *)workspace);
    cudaError_t err = prism::launch_scan_bwd(a, dO, dS_final, dq, dk, gdn ? dv : nullptr, dalpha, dbeta,
                                             gdn ? nullptr : du, gdn ? nullptr : dw, dS0, workspace,
                                             shape->io == PRISM_F32, s);
    probe_finish(s);
    return cuda_status(err);
}

prism_status prism_step_decode(const prism_shape *shape, const void *q, const void *k,
                               const void *v, const float *alpha, const float *beta,
                               const void *u, const void *w, float *S, void *o, void *stream) {
    prism_status st = check_common(shape, q, k, v, alpha, beta, u, w);
    if (st != PRISM_OK) return st;
    if (shape->T != 1) return PRISM_ERR_INVALID_ARG;
    if (shape->dv > 128) return PRISM_ERR_UNSUPPORTED;
    if (shape->B == 0 || shape->H == 0) return PRISM_OK;
    if (!S || !aligned16(S) || !o || !aligned16(o)) return PRISM_ERR_INVALID_ARG;
    if ((long long)shape->B * shape->H > 0x7fffffffLL) return PRISM_ERR_UNSUPPORTED;
    prism::ScanArgs a = make_args(shape, q, k, v, alpha, beta, u, w, nullptr, o, S, nullptr);
    if (g_debug_flags & kDebugStallDecode) a.flags |= prism::kStallDecode;
    cudaError_t err = prism::launch_decode(a, shape->io == PRISM_F32, (cudaStream_t)stream);
    probe_finish((cudaStream_t)stream);
    return cuda_status(err);
}

prism_status prism_write_producer(const prism_shape *shape, const void *x, const void *v,
                                  const float *conv, const void *Wk, const void *Wp,
                                  const float *beta, void *u, void *w, void *stream) {
    if (!shape) return PRISM_ERR_INVALID_ARG;
    const prism_shape &s = *shape;
    if (s.B < 0 || s.H < 0 || s.T < 0 || s.L < 1 || s.dk < 1 || s.dv < 1) return PRISM_ERR_INVALID_ARG;
    if (s.io != PRISM_BF16 && s.io != PRISM_F32) return PRISM_ERR_INVALID_ARG;
    if (s.io != PRISM_BF16 || s.dk != s.dv || (s.dk != 64 && s.dk != 128) || s.L > 64)
        return PRISM_ERR_UNSUPPORTED;
    if (s.B > 65535 || s.H > 65535 || (long long)s.B * s.H > 0x7fffffffLL) return PRISM_ERR_UNSUPPORTED;
    if ((long long)s.B * s.H * s.T == 0) return PRISM_OK;
    for (const void *ptr : {x, v, (const void *)conv, Wk, Wp, (const void *)u, (const void *)w})
        if (!ptr || !aligned16(ptr)) return PRISM_ERR_INVALID_ARG;
    if (!beta || ((uintptr_t)beta & 3u)) return PRISM_ERR_INVALID_ARG;
    for (const void *in : {x, v, (const void *)conv, Wk, Wp, (const void *)beta})
        if (in == u || in == w) return PRISM_ERR_INVALID_ARG;  // outputs alias an input
    if (u == w) return PRISM_ERR_INVALID_ARG;
    prism::ProducerArgs a{s.B, s.H, s.T, s.dk, s.L, x, v, conv, Wk, Wp, beta, u, w,
                          (g_debug_flags & kDebugStallProducer) ? 1 : 0};
    cudaError_t err = prism::launch_write_producer(a, (cudaStream_t)stream);
    probe_finish((cudaStream_t)stream);
    return cuda_status(err);
}

prism_status prism_query_device_status(void *workspace, void *stream) {
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t err = cudaStreamSynchronize(s);
    if (err != cudaSuccess) return cuda_status(err);
    uint32_t word = 0;
    if (workspace) {
        if ((err = cudaMemcpy(&word, workspace, sizeof word, cudaMemcpyDeviceToHost)) != cudaSuccess)
            return cuda_status(err);
        if (word != PRISM_OK && (err = cudaMemset(workspace, 0, sizeof word)) != cudaSuccess)
            return cuda_status(err);
    }
    uint32_t dword = 0, pword = 0, nword = 0;
    if ((err = prism::decode_status(&dword)) != cudaSuccess) return cuda_status(err);
    if ((err = prism::producer_status(&pword)) != cudaSuccess) return cuda_status(err);
    if ((err = prism::noalloc_status(&nword)) != cudaSuccess) return cuda_status(err);
    if (word == PRISM_OK) word = dword;
    if (word == PRISM_OK) word = pword;
    if (word == PRISM_OK) word = nword;
    return (prism_status)word;
}

const char *prism_status_string(prism_status status) {
    switch (status) {
        case PRISM_OK: return "PRISM_OK";
        case PRISM_ERR_INVALID_ARG: return "PRISM_ERR_INVALID_ARG";
        case PRISM_ERR_UNSUPPORTED: return "PRISM_ERR_UNSUPPORTED";
        case PRISM_ERR_CUDA: return "PRISM_ERR_CUDA";
        case PRISM_ERR_TIMEOUT: return "PRISM_ERR_TIMEOUT";
    }
    return "PRISM_ERR_UNKNOWN";
}

const char *prism_last_cuda_error(void) {
    return t_last_cuda_error == cudaSuccess ? "" : cudaGetErrorString(t_last_cuda_error);
}

int prism_debug_set_flags(int flags) {
    int old = g_debug_flags;
    g_debug_flags = flags;
    return old;
}

prism_status prism_debug_record_launch_events(void *const *events, int n_events) {
    if (n_events < 0 || (n_events > 0 && !events)) return PRISM_ERR_INVALID_ARG;
    if (n_events > kMaxProbeEvents) return PRISM_ERR_UNSUPPORTED;
    for (int i = 0; i < n_events; ++i)
        if (!events[i]) return PRISM_ERR_INVALID_ARG;
    t_probe = LaunchProbe{};
    for (int i = 0; i < n_events; ++i) t_probe.events[i] = events[i];
    t_probe.n = n_events;
    return PRISM_OK;
}

}  // extern "C"
