/*
 * prism.h -- C ABI of libprism.so: the gated delta-rule chunked scan forward with a rank-L
 * residual write, and its single-token decode step, on NVIDIA B200 (sm_100a).
 *
 * The operation (per batch b, head h; state S is dv x dk fp32, rows are the value index):
 *
 *     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + sum_{l=1..L} u_{t,l} w_{t,l}^T
 *     o_t = S_t q_t
 *
 * Sources:
 *   - "PRISM: Parallel Residual Iterative Sequence Model" (gist.science explainer), technical
 *     summary section 2.1 (write-forget decoupling: S_t = S_{t-1} A_t + B_t, the forget A_t kept
 *     in Gated-DeltaNet form) and section 2.2 (the rank-L write B_t = sum_l beta^(l) delta^(l)
 *     k^(l)T; here u_{t,l} = beta^(l) delta^(l) and w_{t,l} = k^(l), produced upstream).
 *   - banbantang.com PRISM article, section 1(4): Gated-DeltaNet's scalar decay alpha, rank-1
 *     erase along k and rank-1 write beta v k^T (the L = 1 write used when u, w are NULL).
 *   - "Sequential Parallel Duality in Prefix Scannable Models" (papernotes), key design 2 and the
 *     method overview: each token is an affine element (E_t, f_t) with E_t = alpha_t(I - beta_t
 *     k_t k_t^T), f_t = sum_l u_{t,l} w_{t,l}^T; elements compose associatively, so the sequence
 *     is cut into chunks, each chunk is encoded, and the chunk elements are scanned.
 *
 * Conventions for every entry point:
 *   - Device pointers unless stated otherwise; every buffer is allocated by the caller.  The
 *     library never allocates device or host memory and never synchronises the stream except in
 *     prism_query_device_status.
 *   - Layouts are dense row-major: activations [B,T,H,d]; u [B,T,H,L,dv]; w [B,T,H,L,dk];
 *     alpha, beta [B,T,H]; states [B,H,dv,dk].  alpha and beta must be 4-byte aligned, every
 *     other pointer 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL is the legacy default stream).  All work is
 *     enqueued on it asynchronously.
 *   - Arguments are validated before anything is launched; a rejected call enqueues nothing.
 *     A launch failure returns PRISM_ERR_CUDA.  Kernels never trap: a bounded wait that runs out
 *     records PRISM_ERR_TIMEOUT in the workspace status word (read with
 *     prism_query_device_status).
 *   - Outputs must not alias inputs (except the decode state, which is updated in place).
 */
#ifndef PRISM_H
#define PRISM_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PRISM_OK = 0,
    PRISM_ERR_INVALID_ARG = 1,  /* bad size, NULL pointer, misalignment, short workspace */
    PRISM_ERR_UNSUPPORTED = 2,  /* valid but not built: d not in {32,64,128}, L > 8 ...     */
    PRISM_ERR_CUDA = 3,         /* a CUDA runtime call or kernel launch failed              */
    PRISM_ERR_TIMEOUT = 4       /* a kernel's bounded wait gave up (device status word)     */
} prism_status;

typedef enum { PRISM_BF16 = 0, PRISM_F32 = 1 } prism_dtype;

typedef struct {
    int B, H, T;      /* batch, heads, tokens (T >= 0; decode requires T == 1)              */
    int dk, dv;       /* key and value widths, each in {32, 64, 128}                        */
    int L;            /* write rank, 1..8; must be 1 when u and w are NULL                  */
    int chunk;        /* chunk length of the chunked scan: 64 or 128 (ignored by decode)     */
    prism_dtype io;   /* type of q, k, v, u, w and of o (alpha, beta, states are fp32)      */
} prism_shape;

/*
 * prism_scan_fwd_workspace_size -- bytes of device workspace prism_scan_fwd needs for `shape`
 * (the status word, plus the per-segment affine elements of the segmented scan when B*H is too
 * small to fill the GPU).  Writes *bytes; never fails for a valid shape.
 */
prism_status prism_scan_fwd_workspace_size(const prism_shape *shape, size_t *bytes);

/*
 * prism_scan_fwd_launch_count -- number of kernels one prism_scan_fwd call with `shape` enqueues
 * (the plan depends on B*H, T and the widths).  Host only; writes *launches.
 */
prism_status prism_scan_fwd_launch_count(const prism_shape *shape, int *launches);

/*
 * prism_scan_fwd -- chunked parallel-scan forward over T tokens for all B*H sequences.
 *
 *   q, k     [B,T,H,dk] io     queries and keys (the kernel normalises nothing)
 *   v        [B,T,H,dv] io     values; read only when u == w == NULL (Gated-DeltaNet write
 *                              beta_t v_t k_t^T, requires L == 1); may be NULL otherwise
 *   alpha    [B,T,H] fp32      decay gate, in (0, 1]  (alpha = 0 is outside the domain: the
 *                              chunk form takes log alpha)
 *   beta     [B,T,H] fp32      erase gate
 *   u, w     [B,T,H,L,dv], [B,T,H,L,dk] io, or both NULL: the rank-L write sum_l u w^T
 *   S0       [B,H,dv,dk] fp32  entry state, or NULL for zeros
 *   o        [B,T,H,dv] io     output (bf16 outputs are rounded to nearest even)
 *   S_final  [B,H,dv,dk] fp32  exit state, or NULL to skip; S_final == S0 is allowed
 *   workspace, ws_bytes        device scratch of at least prism_scan_fwd_workspace_size bytes,
 *                              256-byte aligned, zero-filled by the caller before its first
 *                              use (the status word in its first 4 bytes stays zero unless a
 *                              kernel records a failure; prism_query_device_status reads and
 *                              clears it); may be reused once the stream has passed this call
 * The result equals the token recurrence above up to floating-point rounding: state and all
 * accumulation in fp32; bf16 operands are fed to the tensor cores, intermediate results as bf16
 * hi / lo pairs (the chunk's Wk as one bf16 while every state element stays below 4 in
 * magnitude, as a pair once one exceeds it).  Tested against |x - r| <= 2e-2 (1 + |r|) for bf16
 * I/O and 1e-4 (1 + |r|) for fp32 I/O, including write directions of norm ~8 whose state grows
 * into the hundreds.  A partial last chunk is handled as if padded with identity tokens
 * (alpha = 1, beta = 0, no write).
 */
prism_status prism_scan_fwd(const prism_shape *shape, const void *q, const void *k,
                            const void *v, const float *alpha, const float *beta,
                            const void *u, const void *w, const float *S0, void *o,
                            float *S_final, void *workspace, size_t ws_bytes, void *stream);

/*
 * prism_scan_bwd_workspace_size -- bytes of device workspace prism_scan_bwd needs for `shape`:
 * the status block, the state of every (b, h) at each 64-token chunk start, one chunk of states
 * per CTA, and for the chunk-parallel form (bf16 I/O, dk == dv in {64, 128}) the gradient at
 * every chunk end, the reversed token layout and the scans' per-chunk records.  Depends on the
 * current device's SM count.  Writes *bytes.
 */
prism_status prism_scan_bwd_workspace_size(const prism_shape *shape, size_t *bytes);

/*
 * prism_scan_bwd -- the backward pass of prism_scan_fwd: given the forward's inputs and the
 * upstream gradients dO of o and dS_final of S_final, the gradients of every input, for training
 * ("PRISM: Parallel Residual Iterative Sequence Model", gist.science explainer, section 4: the
 * method's throughput is training throughput; the recurrence of technical summary 2.1-2.2).  With
 * G_t the gradient of S_t (G_T = dS_final), running from the last token to the first:
 *   G_t += dO_t q_t^T;   dq_t = S_t^T dO_t;
 *   dalpha_t = <G_t, S_{t-1}(I - beta_t k_t k_t^T)>;
 *   dbeta_t = -alpha_t (S_{t-1}k_t).(G_t k_t)  (+ v_t.(G_t k_t) for the GDN write);
 *   dk_t = -alpha_t beta_t (G_t^T S_{t-1}k_t + S_{t-1}^T G_t k_t)  (+ beta_t G_t^T v_t);
 *   dv_t = beta_t G_t k_t  (GDN write)  |  du_{t,l} = G_t w_{t,l},  dw_{t,l} = G_t^T u_{t,l};
 *   G_{t-1} = alpha_t G_t (I - beta_t k_t k_t^T);   dS0 = G_0.
 *   q, k, v, alpha, beta, u, w, S0   exactly as passed to prism_scan_fwd (same shape rules)
 *   dO        [B,T,H,dv] io       upstream gradient of o
 *   dS_final  [B,H,dv,dk] fp32    upstream gradient of S_final, or NULL for zero
 *   dq, dk    [B,T,H,dk] fp32     outputs (gradients are fp32 whatever the I/O type)
 *   dv        [B,T,H,dv] fp32     output, GDN write only (ignored on the rank-L write)
 *   dalpha, dbeta [B,T,H] fp32    outputs
 *   du, dw    [B,T,H,L,dv], [B,T,H,L,dk] fp32   outputs, rank-L write only (ignored otherwise)
 *   dS0       [B,H,dv,dk] fp32    output, or NULL to skip
 *   workspace, ws_bytes           at least prism_scan_bwd_workspace_size bytes, 256-byte aligned
 * Every pointer 16-byte aligned; no gradient may overlap another or an input.  With bf16 I/O and
 * dk == dv in {64, 128} the work is chunk-parallel: the forward scan's tensor-core kernels write
 * every 64-token chunk's entry state and, run over the reversed tokens with the rank-1 write
 * dO q^T, the gradient at every chunk end (and dS0); every chunk's token-level reverse pass then
 * runs on its own, in fp32 on CUDA cores.  Otherwise each CTA re-runs the forward recurrence for
 * its value rows (checkpointing every 64 tokens) and walks the tokens backwards chunk by chunk,
 * all in fp32 on CUDA cores from the exact input values.
 * dq, dk, dw, dalpha and dbeta are sums over value rows accumulated with atomic adds (cleared on
 * the stream first), so their last bits depend on the order of those adds.  Tested against
 * |x - r| <= tol (1 + |r|) with tol = 2e-2 (bf16 I/O) and 1e-4 (fp32 I/O).
 */
prism_status prism_scan_bwd(const prism_shape *shape, const void *q, const void *k, const void *v,
                            const float *alpha, const float *beta, const void *u, const void *w,
                            const float *S0, const void *dO, const float *dS_final, float *dq,
                            float *dk, float *dv, float *dalpha, float *dbeta, float *du, float *dw,
                            float *dS0, void *workspace, size_t ws_bytes, void *stream);

/*
 * prism_scan_segment_element -- the affine map of a token segment, the building block of a scan
 * split across devices along T ("Sequential Parallel Duality in Prefix Scannable Models", method
 * overview: every chunk is an element of an associative operator and elements compose in order).
 * For every (b, h), the recurrence over the segment sends any entry state S to  S E + f  with
 *   E        [B,H,dk,dk] fp32  the product of the per-token transitions alpha_t (I - beta_t k_t k_t^T)
 *   f        [B,H,dv,dk] fp32  the exit state from S = 0 (the writes carried to the segment end)
 * Requires dk == dv.  Other arguments, the workspace and the rounding are as for prism_scan_fwd
 * (no S0, no outputs).  E and f must not overlap.
 */
prism_status prism_scan_segment_element(const prism_shape *shape, const void *q, const void *k,
                                        const void *v, const float *alpha, const float *beta,
                                        const void *u, const void *w, float *E, float *f,
                                        void *workspace, size_t ws_bytes, void *stream);

/*
 * prism_state_fold -- S_out = S_in E + f for each of BH states (the element composition of
 * prism_scan_segment_element applied to a state): S_in, f, S_out [BH,dv,dk] fp32, E [BH,dk,dk]
 * fp32; S_in NULL means zero (S_out = f); S_out may be S_in but not E or f.  fp32 on CUDA cores.
 * dk, dv in {32, 64, 128}.
 */
prism_status prism_state_fold(int BH, int dk, int dv, const float *S_in, const float *E,
                              const float *f, float *S_out, void *stream);

/*
 * prism_step_decode -- one token for each of the B*H sequences (shape->T must be 1):
 *   S <- alpha S (I - beta k k^T) + sum_l u_l w_l^T   (in place),   o = S q.
 * Arguments as for prism_scan_fwd with T == 1; S is read and written in place, [B,H,dv,dk]
 * fp32; o is [B,1,H,dv] io.  A pure HBM-bound rank-(L+1) update: one read and one write of S.
 */
prism_status prism_step_decode(const prism_shape *shape, const void *q, const void *k,
                               const void *v, const float *alpha, const float *beta,
                               const void *u, const void *w, float *S, void *o, void *stream);

/*
 * prism_scan_fwd_noalloc -- prism_scan_fwd for callers that cannot allocate device memory when
 * they run the scan (for example a plugin inside an engine that owns all device allocations, or
 * a latency-critical path that cannot afford cudaMalloc's implicit synchronisation).  Same
 * arguments and results as prism_scan_fwd, minus the workspace: the library uses its own
 * scratch, a fixed PRISM_NOALLOC_SCRATCH_BYTES array in device global memory that every GPU which
 * loads libprism.so holds until the process exits.  This call allocates nothing.
 *   - Shapes whose workspace (prism_scan_fwd_workspace_size) exceeds PRISM_NOALLOC_SCRATCH_BYTES
 *     are rejected with PRISM_ERR_UNSUPPORTED before anything is enqueued.
 *   - Arguments are checked as prism_scan_fwd checks them, with the same status codes, before
 *     anything is sized or enqueued.
 *   - The first call on each device looks up the scratch's device address (with that device
 *     current) and caches it, and looks it up again if the device's context has changed (after
 *     a cudaDeviceReset); make that first call before any stream capture.
 *   - All calls on a device share the one scratch array, which keeps the last call's contents:
 *     calls whose kernels overlap on the GPU (different streams, no ordering between them) race
 *     on it.  Serialise them (one stream, or events).
 *   - The scratch's first 4 bytes are the scan's status word (zero when the library loads): a
 *     kernel whose bounded wait gave up records PRISM_ERR_TIMEOUT there, and
 *     prism_query_device_status(NULL, stream), called with the same device current, reports
 *     and clears it.
 * The method pages have no counterpart of this entry point; it exists for the callers above.
 */
#define PRISM_NOALLOC_SCRATCH_BYTES (16u << 20)
prism_status prism_scan_fwd_noalloc(const prism_shape *shape, const void *q, const void *k,
                                    const void *v, const float *alpha, const float *beta,
                                    const void *u, const void *w, const float *S0, void *o,
                                    float *S_final, void *stream);

/*
 * prism_write_producer -- the input-anchored write terms in front of the scan ("PRISM: Parallel
 * Residual Iterative Sequence Model", gist.science explainer, technical summary 2.2; the anchor
 * width of the banbantang.com PRISM article, section 5(1), the first residual of its section
 * 3(4)).  For every (b, t, h), with d = dk = dv:
 *   a_t     = sum_{j=0..3} conv[h][j] * x_{t-j}            depthwise causal ShortConv, x_{<0} = 0
 *   k^(l)   = Wk[h][l] a_t,   p^(l) = Wp[h][l] a_t          l = 1..L (row = output index)
 *   r^(1)   = v_t,   delta^(l) = GELU(p^(l) * r^(l)),   r^(l+1) = r^(l) - delta^(l)   (exact GELU)
 *   u_{t,l} = beta_t^(l) delta^(l),   w_{t,l} = k^(l)
 * so that prism_scan_fwd with these u, w writes B_t = sum_l beta delta k^T.
 *   x, v     [B,T,H,d]   bf16          conv  [H,4,d]  fp32 (conv[h][0] multiplies x_t)
 *   Wk, Wp   [H,L,d,d]   bf16          beta  [B,T,H,L] fp32 (4-byte aligned)
 *   u, w     [B,T,H,L,d] bf16 outputs  (must not overlap each other or any input)
 * Uses shape->B, H, T, dk, dv, L, io; requires io == PRISM_BF16 and dk == dv in {64, 128}
 * (PRISM_ERR_UNSUPPORTED otherwise), 1 <= L <= 64, B <= 65535, H <= 65535 and B * H < 2^31.
 * The two projections run on the tensor cores from the anchor as a bf16 hi / lo pair with fp32
 * accumulation; the residual chain and GELU in fp32, GELU's erf by Abramowitz & Stegun, Handbook
 * of Mathematical Functions, 7.1.26 (absolute error at most 1.5e-7); u, w are rounded to bf16
 * (nearest even).  A bounded wait that gives up records PRISM_ERR_TIMEOUT in the library's
 * producer status word (prism_query_device_status).
 */
prism_status prism_write_producer(const prism_shape *shape, const void *x, const void *v,
                                  const float *conv, const void *Wk, const void *Wp,
                                  const float *beta, void *u, void *w, void *stream);

/*
 * prism_query_device_status -- synchronise `stream`, read the status word in `workspace` (written
 * by scan kernels whose bounded waits ran out; workspace may be NULL) and the library's own
 * status words on the current device (decode, producer, and the scratch of
 * prism_scan_fwd_noalloc), and clear them.  Returns PRISM_OK, PRISM_ERR_TIMEOUT, or
 * PRISM_ERR_CUDA if the stream itself reports an error.
 */
prism_status prism_query_device_status(void *workspace, void *stream);

/* prism_status_string -- a static, human-readable name for a status code. */
const char *prism_status_string(prism_status status);

/*
 * prism_last_cuda_error -- the CUDA runtime's description of the error behind the calling host
 * thread's most recent PRISM_ERR_CUDA ("" if there was none).  Static storage; never NULL.
 */
const char *prism_last_cuda_error(void);

/*
 * prism_debug_set_flags -- testing and measurement hook (process-wide; set it before
 * prism_scan_fwd_workspace_size, which depends on it).  flags bit 1: prism_scan_fwd takes the
 * segmented inter-chunk scan (segment elements, a Blelloch scan over them, a re-run of every
 * segment) whenever the shape allows it (dk == dv, T divisible into segments of >= 64 tokens);
 * bit 2: it never does; bit 3: the stall test -- the Gated-DeltaNet state kernel's load warp
 * issues nothing, every wait gives up after a short limit, the kernel records PRISM_ERR_TIMEOUT
 * in the workspace status word and returns (outputs are then undefined); bit 4: the tensor-core
 * state kernel applies its Wk_lo precision term from the first chunk instead of only once the
 * state has grown large (results stay within the same tolerance); bits 5, 6, 7: the same stall
 * test for the per-chunk prep kernels of the tensor-core scan (their tile loads are not issued;
 * PRISM_ERR_TIMEOUT in the workspace status word), for prism_write_producer (its weight loads;
 * the producer status word) and for the bulk-copy decode kernel (its state copies; the decode
 * status word).  Returns the previous flags.
 */
int prism_debug_set_flags(int flags);

/*
 * prism_debug_record_launch_events -- measurement hook.  Arms the calling host thread's next
 * prism_scan_fwd or prism_step_decode call to record events[j] (cudaEvent_t handles owned by the
 * caller, created on the stream's device) on its stream right before its kernel launch j, and one
 * more event after its last launch, for as many events as n_events allows (a call makes
 * prism_scan_fwd_launch_count() launches, so n_events = launches + 1 brackets every one).  The
 * probe is disarmed by that call, whatever it returns; n_events = 0 disarms it.  The handles are
 * copied: the array need not outlive this call, the events must outlive the probed call.  Event
 * record errors are not reported.  Returns PRISM_ERR_INVALID_ARG if n_events < 0 or a handle is
 * NULL, PRISM_ERR_UNSUPPORTED if n_events > 64.
 */
prism_status prism_debug_record_launch_events(void *const *events, int n_events);

#ifdef __cplusplus
}
#endif
#endif /* PRISM_H */
