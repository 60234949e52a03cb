"""fp64 oracle for the backward pass of the scan (gradients of every input).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import this module.  It shares no code with the CUDA library.

The forward is the token recurrence of "PRISM: Parallel Residual Iterative Sequence Model"
(gist.science explainer, technical summary 2.1 and 2.2; banbantang.com PRISM article, section
1(4) for the Gated-DeltaNet forget and write):

    S_t = alpha_t S_{t-1} A_t + W_t,   A_t = I - beta_t k_t k_t^T,   o_t = S_t q_t
    W_t = beta_t v_t k_t^T  (the GDN write, u and w absent)  or  sum_l u_{t,l} w_{t,l}^T

For a scalar loss with upstream gradients do_t (of o_t) and dS_T (of the exit state), the
gradient G_t of S_t obeys, from t = T down to 1 (G_T starts at dS_T):

    G_t   += do_t q_t^T                                (o_t reads S_t)
    dq_t   = S_t^T do_t
    dalpha_t = <G_t, S_{t-1} A_t>
    dbeta_t  = -alpha_t (S_{t-1} k_t) . (G_t k_t)       (+ v_t . (G_t k_t) for the GDN write)
    dk_t   = -alpha_t beta_t (G_t^T S_{t-1} k_t + S_{t-1}^T G_t k_t)   (+ beta_t G_t^T v_t, GDN)
    dv_t   = beta_t G_t k_t                             (GDN write)
    du_{t,l} = G_t w_{t,l},   dw_{t,l} = G_t^T u_{t,l}  (rank-L write)
    G_{t-1} = alpha_t G_t A_t^T = alpha_t (G_t - beta_t (G_t k_t) k_t^T)

and dS0 = G_0.  One token at a time, with the states of the forward kept; the pins
(``tests/test_grad_pins.py``) compare every gradient with central finite differences of the
forward oracle (``oracle.scan_ref``, a separate C implementation).
"""
from __future__ import annotations

import numpy as np


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):
        return a.detach().to("cpu").double().numpy()
    return np.asarray(a, dtype=np.float64)


def scan_grad_ref(q, k, v, alpha, beta, u=None, w=None, S0=None, *, do, dS_final=None, mutant=0):
    """Inputs as for ``oracle.scan_ref`` (q, k [B,T,H,dk]; v [B,T,H,dv] or None; alpha, beta
    [B,T,H]; u [B,T,H,L,dv] and w [B,T,H,L,dk] or None; S0 [B,H,dv,dk] or None), do [B,T,H,dv],
    dS_final [B,H,dv,dk] or None.  Returns a dict of fp64 gradients with the inputs' shapes:
    dq, dk, dv (None on the rank-L write), dalpha, dbeta, du, dw (None on the GDN write), dS0.

    ``mutant`` plants one mistake, for the pin tests only: 1 the state gradient is carried back
    without alpha; 2 dk keeps only one of its two symmetric terms; 3 dq reads S_{t-1}."""
    q, k, v, alpha, beta, u, w, S0, do, dS_final = map(_f64, (q, k, v, alpha, beta, u, w, S0, do, dS_final))
    B, T, H, dk = q.shape
    gdn = u is None
    dv_ = v.shape[-1] if gdn else u.shape[-1]
    out = {n: np.zeros_like(x) for n, x in (("dq", q), ("dk", k), ("dalpha", alpha), ("dbeta", beta))}
    out["dv"] = np.zeros_like(v) if gdn else None
    out["du"] = None if gdn else np.zeros_like(u)
    out["dw"] = None if gdn else np.zeros_like(w)
    out["dS0"] = np.zeros((B, H, dv_, dk))
    eye = np.eye(dk)
    for b in range(B):
        for h in range(H):
            S = np.zeros((dv_, dk)) if S0 is None else S0[b, h].copy()
            states = [S]
            for t in range(T):
                kt = k[b, t, h]
                A = eye - beta[b, t, h] * np.outer(kt, kt)
                if gdn:
                    W = beta[b, t, h] * np.outer(v[b, t, h], kt)
                else:
                    W = sum(np.outer(u[b, t, h, l], w[b, t, h, l]) for l in range(u.shape[3]))
                S = alpha[b, t, h] * states[-1] @ A + W
                states.append(S)
            G = np.zeros((dv_, dk)) if dS_final is None else dS_final[b, h].copy()
            for t in reversed(range(T)):
                kt, a_t, b_t = k[b, t, h], alpha[b, t, h], beta[b, t, h]
                St, P = states[t + 1], states[t]
                G = G + np.outer(do[b, t, h], q[b, t, h])
                out["dq"][b, t, h] = (P if mutant == 3 else St).T @ do[b, t, h]
                Pk, Gk = P @ kt, G @ kt
                A = eye - b_t * np.outer(kt, kt)
                out["dalpha"][b, t, h] = np.sum(G * (P @ A))
                dbeta = -a_t * Pk @ Gk
                dkt = -a_t * b_t * (G.T @ Pk + (0 if mutant == 2 else P.T @ Gk))
                if gdn:
                    vt = v[b, t, h]
                    out["dv"][b, t, h] = b_t * Gk
                    dbeta += vt @ Gk
                    dkt += b_t * (G.T @ vt)
                else:
                    for l in range(u.shape[3]):
                        out["du"][b, t, h, l] = G @ w[b, t, h, l]
                        out["dw"][b, t, h, l] = G.T @ u[b, t, h, l]
                out["dbeta"][b, t, h] = dbeta
                out["dk"][b, t, h] = dkt
                G = (1.0 if mutant == 1 else a_t) * (G - b_t * np.outer(Gk, kt))
            out["dS0"][b, h] = G
    return out
