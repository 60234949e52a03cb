/*
 * prism_ref.c -- fp64 CPU oracle for the gated delta-rule scan with a rank-L write.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness reference that the GPU library is
 * checked against.  It shares no code, header, table or helper with the CUDA path and must
 * never be linked into it; only the tests, the package smoke check and the CPU-baseline leg
 * of the bench load it.
 *
 * What it computes (plain definition, token by token, in double precision):
 *
 *   per (batch b, head h), with state S in R^{dv x dk} (rows = value index):
 *     S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T)  +  sum_{l=1..L} u_{t,l} w_{t,l}^T
 *     o_t = S_t q_t
 *
 *   Sources:
 *   - "PRISM: Parallel Residual Iterative Sequence Model" (gist.science explainer), technical
 *     summary section 2.1 "Write-Forget Decoupling": the update is S_t = S_{t-1} A_t + B_t,
 *     with the forget operator A_t kept in Gated-DeltaNet form.
 *   - same page, section 2.2 "Input-Anchored Loop Unrolling": the write is a rank-L sum of
 *     outer products B_t = sum_l beta^(l) delta^(l) (k^(l))^T; here u_{t,l} carries
 *     beta^(l) delta^(l) (the per-step gate is folded into u by its producer) and w_{t,l}
 *     carries the direction k^(l).
 *   - banbantang.com PRISM article, section 1(4) "the rank-1 write bottleneck": the GDN form,
 *     a global scalar gate alpha for decay, a rank-1 selective erase (I - beta k k^T) along k
 *     and the rank-1 write beta v k^T.  With u == NULL and w == NULL this file uses exactly
 *     that write (L must be 1): S_t = alpha_t S_{t-1}(I - beta_t k_t k_t^T) + beta_t v_t k_t^T.
 *
 *   Readings taken where the pages are silent (each listed in the design notes):
 *   - alpha multiplies only the forget term; the write of step t is not decayed in step t.
 *   - the output reads the post-update state S_t.
 *   - no 1/sqrt(dk) scaling of q; nothing is normalised here.
 *   - layouts: activations [B,T,H,...] row-major; state [B,H,dv,dk] row-major.
 *
 * Inputs are the exact values the GPU receives (bf16 bit patterns or fp32), widened to double
 * without rounding.  alpha, beta are fp32 [B,T,H].  u is [B,T,H,L,dv], w is [B,T,H,L,dk].
 *
 * Parity pins: every function here is pinned by host tests against closed forms (causal
 * linear attention, gated linear attention), the delta-rule overwrite identity, a brute-force
 * Blelloch scan over explicit affine elements, superposition, row independence and
 * resumability.  No function here is unpinned.
 *
 * The mutant entry point exists only so that tests can plant a known mistake in the oracle
 * and confirm that at least one pin catches it.
 */
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "../include/prism_ref.h"

/* Widen one input element to double.  bf16 is the upper half of an IEEE binary32, so the
 * widening is exact: shift the 16 bits into the high half of a float. */
static double load_io(const void *p, size_t i, int io_f32)
{
    if (io_f32) {
        return (double)((const float *)p)[i];
    }
    uint32_t bits = ((uint32_t)((const uint16_t *)p)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

typedef struct {
    int B, H, T, dk, dv, L, io_f32, mutation;
    const void *q, *k, *v, *u, *w;
    const float *alpha, *beta;
    const double *S0;
    double *o, *S_final;
    int next_job; /* shared counter over (b,h) jobs, guarded by lock */
    pthread_mutex_t lock;
} ref_job;

/* One (b,h) sequence, token by token. */
static void run_head(const ref_job *J, int b, int h, double *S, double *kt, double *qt,
                     double *e, double *tmp)
{
    const int dk = J->dk, dv = J->dv, L = J->L, H = J->H, T = J->T;
    const size_t head = (size_t)b * H + h;

    if (J->S0) {
        memcpy(S, J->S0 + head * dv * dk, sizeof(double) * dv * dk);
    } else {
        memset(S, 0, sizeof(double) * dv * dk);
    }

    for (int t = 0; t < T; ++t) {
        const size_t bth = ((size_t)b * T + t) * H + h; /* index of (b,t,h) */
        const double a = (double)J->alpha[bth];
        const double be = (double)J->beta[bth];
        for (int j = 0; j < dk; ++j) {
            kt[j] = load_io(J->k, bth * dk + j, J->io_f32);
            qt[j] = load_io(J->q, bth * dk + j, J->io_f32);
        }

        if (J->mutation == 5) {
            /* mutant: readout taken from the pre-update state S_{t-1} */
            for (int r = 0; r < dv; ++r) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += S[(size_t)r * dk + j] * qt[j];
                J->o[bth * dv + r] = acc;
            }
        }

        /* e = S_{t-1} k_t  (the part of the old state along k_t) */
        for (int r = 0; r < dv; ++r) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[(size_t)r * dk + j] * kt[j];
            e[r] = acc;
        }

        /* forget: S <- alpha (S - beta e k^T) = alpha S (I - beta k k^T) */
        for (int r = 0; r < dv; ++r) {
            for (int j = 0; j < dk; ++j) {
                double s = S[(size_t)r * dk + j];
                double erase = be * e[r] * kt[j];
                if (J->mutation == 1) erase = 0.0;          /* mutant: erase dropped      */
                if (J->mutation == 2) erase = -erase;       /* mutant: erase sign flipped */
                S[(size_t)r * dk + j] = a * (s - erase);
            }
        }

        /* write: + sum_l u_{t,l} w_{t,l}^T, or the GDN write beta v k^T */
        if (J->u == NULL) {
            for (int r = 0; r < dv; ++r) {
                double vr = load_io(J->v, bth * dv + r, J->io_f32);
                double scale = (J->mutation == 3) ? a * be : be; /* mutant: write decayed */
                for (int j = 0; j < dk; ++j) S[(size_t)r * dk + j] += scale * vr * kt[j];
            }
        } else {
            for (int l = 0; l < L; ++l) {
                const size_t ub = (bth * L + l) * dv;
                const size_t wb = (bth * L + l) * dk;
                for (int j = 0; j < dk; ++j) tmp[j] = load_io(J->w, wb + j, J->io_f32);
                for (int r = 0; r < dv; ++r) {
                    double ur = load_io(J->u, ub + r, J->io_f32);
                    if (J->mutation == 4 && l > 0) ur = 0.0; /* mutant: only first write */
                    if (J->mutation == 7) ur *= a;           /* mutant: write decayed      */
                    for (int j = 0; j < dk; ++j) {
                        double wj = tmp[j];
                        if (J->mutation == 6 && dk == dv) {
                            /* mutant: outer product transposed, w u^T instead of u w^T */
                            wj = load_io(J->u, ub + j, J->io_f32);
                            ur = tmp[r];
                        }
                        S[(size_t)r * dk + j] += ur * wj;
                    }
                }
            }
        }

        /* readout: o_t = S_t q_t (post-update state) */
        if (J->mutation != 5) {
            for (int r = 0; r < dv; ++r) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += S[(size_t)r * dk + j] * qt[j];
                J->o[bth * dv + r] = acc;
            }
        }
    }

    if (J->S_final) memcpy(J->S_final + head * dv * dk, S, sizeof(double) * dv * dk);
}

static void *worker(void *arg)
{
    ref_job *J = (ref_job *)arg;
    const int dk = J->dk, dv = J->dv;
    double *S = (double *)malloc(sizeof(double) * ((size_t)dv * dk + 3 * (size_t)dk + dv));
    if (!S) return NULL;
    double *kt = S + (size_t)dv * dk;
    double *qt = kt + dk;
    double *tmp = qt + dk;
    double *e = tmp + dk;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int job = J->next_job++;
        pthread_mutex_unlock(&J->lock);
        if (job >= J->B * J->H) break;
        run_head(J, job / J->H, job % J->H, S, kt, qt, e, tmp);
    }
    free(S);
    return NULL;
}

static int scan_ref_impl(int B, int H, int T, int dk, int dv, int L, int io_f32,
                         const void *q, const void *k, const void *v, const float *alpha,
                         const float *beta, const void *u, const void *w, const double *S0,
                         double *o_out, double *S_final_out, int n_threads, int mutation)
{
    if (B < 0 || H < 0 || T < 0 || dk < 1 || dv < 1 || L < 1) return PRISM_REF_ERR_INVALID_ARG;
    if ((u == NULL) != (w == NULL)) return PRISM_REF_ERR_INVALID_ARG;
    if (u == NULL && (L != 1 || v == NULL)) return PRISM_REF_ERR_INVALID_ARG;
    if (T > 0 && (q == NULL || k == NULL || alpha == NULL || beta == NULL || o_out == NULL))
        return PRISM_REF_ERR_INVALID_ARG;
    if (B == 0 || H == 0) return PRISM_REF_OK;

    ref_job J;
    memset(&J, 0, sizeof J);
    J.B = B; J.H = H; J.T = T; J.dk = dk; J.dv = dv; J.L = L; J.io_f32 = io_f32;
    J.mutation = mutation;
    J.q = q; J.k = k; J.v = v; J.u = u; J.w = w; J.alpha = alpha; J.beta = beta; J.S0 = S0;
    J.o = o_out; J.S_final = S_final_out;
    pthread_mutex_init(&J.lock, NULL);

    int nt = n_threads < 1 ? 1 : n_threads;
    if (nt > B * H) nt = B * H;
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nt);
    if (!tid) return PRISM_REF_ERR_INVALID_ARG;
    int started = 0;
    for (int i = 0; i + 1 < nt; ++i) {
        if (pthread_create(&tid[started], NULL, worker, &J) == 0) ++started;
    }
    worker(&J); /* the calling thread works too */
    for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
    free(tid);
    pthread_mutex_destroy(&J.lock);
    return PRISM_REF_OK;
}

int prism_scan_ref(int B, int H, int T, int dk, int dv, int L, int io_f32, const void *q,
                   const void *k, const void *v, const float *alpha, const float *beta,
                   const void *u, const void *w, const double *S0, double *o_out,
                   double *S_final_out, int n_threads)
{
    return scan_ref_impl(B, H, T, dk, dv, L, io_f32, q, k, v, alpha, beta, u, w, S0, o_out,
                         S_final_out, n_threads, 0);
}

int prism_scan_ref_mutant(int B, int H, int T, int dk, int dv, int L, int io_f32,
                          const void *q, const void *k, const void *v, const float *alpha,
                          const float *beta, const void *u, const void *w, const double *S0,
                          double *o_out, double *S_final_out, int n_threads, int mutation)
{
    return scan_ref_impl(B, H, T, dk, dv, L, io_f32, q, k, v, alpha, beta, u, w, S0, o_out,
                         S_final_out, n_threads, mutation);
}
