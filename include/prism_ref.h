/*
 * prism_ref.h -- C ABI of the fp64 CPU oracle (liboracle_prism.so, built from oracle/).
 *
 * TEST INFRASTRUCTURE.  This library is the correctness reference for libprism.so.  It is a
 * separate shared object that shares no code or header with the CUDA library; only tests,
 * the package smoke check and the CPU-baseline leg of the bench load it.
 *
 * Operation (per batch b, head h; state S is dv x dk, rows are the value index):
 *     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + sum_{l=1..L} u_{t,l} w_{t,l}^T
 *     o_t = S_t q_t
 * Defined by "PRISM: Parallel Residual Iterative Sequence Model" (gist.science explainer),
 * technical summary sections 2.1 (write-forget decoupling, S_t = S_{t-1} A_t + B_t with A_t
 * in Gated-DeltaNet form) and 2.2 (rank-L write B_t = sum_l beta^(l) delta^(l) k^(l)T), and
 * by the banbantang.com PRISM article, section 1(4) (the GDN forget and rank-1 write).
 */
#ifndef PRISM_REF_H
#define PRISM_REF_H

#ifdef __cplusplus
extern "C" {
#endif

enum { PRISM_REF_OK = 0, PRISM_REF_ERR_INVALID_ARG = 1 };

/*
 * prism_scan_ref -- token-by-token recurrence in double precision.  All pointers are HOST.
 *
 *   B, H, T, dk, dv, L : sizes; B, H, T >= 0; dk, dv, L >= 1.
 *   io_f32             : 1 if q, k, v, u, w hold fp32; 0 if they hold bf16 bit patterns
 *                        (uint16).  Values are widened to double exactly.
 *   q, k               : [B,T,H,dk]   v : [B,T,H,dv] (only read when u == NULL)
 *   alpha, beta        : fp32 [B,T,H]; alpha is the decay gate, beta the erase gate.
 *   u, w               : [B,T,H,L,dv] and [B,T,H,L,dk], or both NULL.  Both NULL selects
 *                        the Gated-DeltaNet write beta_t v_t k_t^T and requires L == 1.
 *   S0                 : double [B,H,dv,dk] entry state, or NULL for zeros.
 *   o_out              : double [B,T,H,dv], written.
 *   S_final_out        : double [B,H,dv,dk], written; may be NULL.
 *   n_threads          : worker threads over (b,h) pairs (the caller counts as one).
 * Returns PRISM_REF_OK, or PRISM_REF_ERR_INVALID_ARG (nothing written) for bad sizes or a
 * NULL pointer that the arguments require.  The caller owns every buffer.
 */
int prism_scan_ref(int B, int H, int T, int dk, int dv, int L, int io_f32, const void *q,
                   const void *k, const void *v, const float *alpha, const float *beta,
                   const void *u, const void *w, const double *S0, double *o_out,
                   double *S_final_out, int n_threads);

/*
 * prism_scan_ref_mutant -- the same recurrence with one deliberate mistake planted, so the
 * host tests can show that the oracle's pins catch it.  mutation: 0 none; 1 erase dropped;
 * 2 erase sign flipped; 3 GDN write decayed by alpha; 4 only the first of L writes kept;
 * 5 readout from the pre-update state; 6 write outer product transposed (dk == dv);
 * 7 rank-L write decayed by alpha.  Never used outside tests.
 */
int prism_scan_ref_mutant(int B, int H, int T, int dk, int dv, int L, int io_f32,
                          const void *q, const void *k, const void *v, const float *alpha,
                          const float *beta, const void *u, const void *w, const double *S0,
                          double *o_out, double *S_final_out, int n_threads, int mutation);

#ifdef __cplusplus
}
#endif
#endif /* PRISM_REF_H */
