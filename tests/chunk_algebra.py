"""fp64 numpy mirror of the chunked (WY / UT-transform) form of the scan.

Test helper: it is not the oracle and the CUDA path does not use it.  It writes out, in plain
numpy, the per-chunk algebra that the GPU kernels implement, so that the derivation itself can be
checked against the token-by-token oracle for many chunk sizes, separately from any kernel.

Per head, chunk of n tokens (indices t, i within the chunk), entry state S (dv x dk):
  g_t = sum_{r<=t} log alpha_r,  gamma_t = exp(g_t),  Gamma_{t,i} = exp(g_t - g_i)
  x_t := alpha_t beta_t S_{t-1} k_t  turns the recurrence into
      S_t = alpha_t S_{t-1} - x_t k_t^T + sum_l u_{t,l} w_{t,l}^T
  and solving for the x_t of the chunk gives (I + A) X = diag(beta gamma) K S^T + P U~ with
      A_{t,i} = beta_t Gamma_{t,i} k_t.k_i            (i < t)
      P_{t,(i,l)} = beta_t Gamma_{t,i} k_t.w_{i,l}     (i < t)
  so with T = (I + A)^{-1}:  X = Wk S^T + X_u,  Wk = T diag(beta gamma) K,  X_u = T P U~.
  Outputs:  O = diag(gamma) Q S^T - Mqk X + Mqw U~,  Mqk_{t,i} = Gamma_{t,i} q_t.k_i (i <= t),
            Mqw_{t,(i,l)} = Gamma_{t,i} q_t.w_{i,l} (i <= t)
  Exit state: S' = gamma_n S - X^T D K + U~^T D~ W~,  D = diag(gamma_n / gamma_i).
  Affine element of the chunk: S' = S E_c + f_c with E_c = gamma_n I - Wk^T D K and
  f_c = U~^T D~ W~ - X_u^T D K.
Gated-DeltaNet write (u = beta v, w = k): with U_ps = T diag(beta) V and Y = U_ps - Wk S^T,
  O = diag(gamma) Q S^T + Mqk Y  and  S' = gamma_n S + Y^T D K.
"""
from __future__ import annotations

import numpy as np


def _to64(x):
    if x is None:
        return None
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().cpu().double().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def chunk_terms(Kc, Qc, ac, bc, Uc, Wc):
    """State-independent terms of one chunk.  Kc, Qc: n x dk; ac, bc: n; Uc: n x L x dv;
    Wc: n x L x dk.  Returns a dict of the quantities named in the module docstring."""
    n = Kc.shape[0]
    L = Uc.shape[1]
    g = np.cumsum(np.log(ac))
    gam = np.exp(g)
    Gam = np.exp(g[:, None] - g[None, :])
    strict = np.tril(np.ones((n, n)), -1)
    incl = np.tril(np.ones((n, n)))
    A = strict * (bc[:, None] * (Kc @ Kc.T) * Gam)
    Tm = np.linalg.inv(np.eye(n) + A)
    Wk = Tm @ ((bc * gam)[:, None] * Kc)
    Ut = Uc.reshape(n * L, -1)                 # rows ordered (i, l)
    Wt = Wc.reshape(n * L, -1)
    KW = (Kc @ Wt.T).reshape(n, n, L)          # [t, i, l] = k_t . w_{i,l}
    QW = (Qc @ Wt.T).reshape(n, n, L)
    P = (bc[:, None, None] * Gam[:, :, None] * strict[:, :, None] * KW).reshape(n, n * L)
    Mqw = (Gam[:, :, None] * incl[:, :, None] * QW).reshape(n, n * L)
    Mqk = incl * (Qc @ Kc.T) * Gam
    Xu = Tm @ (P @ Ut)
    D = np.exp(g[-1] - g)                      # gamma_n / gamma_i
    Dt = np.repeat(D, L)
    return dict(g=g, gam=gam, Gam=Gam, A=A, T=Tm, Wk=Wk, P=P, Mqk=Mqk, Mqw=Mqw, Xu=Xu, D=D,
                Dt=Dt, Ut=Ut, Wt=Wt)


def chunk_element(Kc, terms, dv):
    """(E_c, f_c) of one chunk: S' = S E_c + f_c."""
    dk = Kc.shape[1]
    tm = terms
    E = tm["gam"][-1] * np.eye(dk) - tm["Wk"].T @ (tm["D"][:, None] * Kc)
    f = tm["Ut"].T @ (tm["Dt"][:, None] * tm["Wt"]) - tm["Xu"].T @ (tm["D"][:, None] * Kc)
    return E, f


def chunked_forward(q, k, v, alpha, beta, u=None, w=None, S0=None, chunk=64, gdn_fused=False):
    """Chunked evaluation of the scan.  Same argument layout as the oracle.  Returns
    (o [B,T,H,dv], S_final [B,H,dv,dk]) in float64.  gdn_fused selects the Gated-DeltaNet
    form (requires u, w None)."""
    q, k, v, alpha, beta = map(_to64, (q, k, v, alpha, beta))
    u, w, S0 = _to64(u), _to64(w), _to64(S0)
    B, T, H, dk = q.shape
    if u is None:
        dv = v.shape[3]
        u = (beta[..., None] * v)[:, :, :, None, :]
        w = k[:, :, :, None, :]
    else:
        dv = u.shape[4]
        if gdn_fused:
            raise ValueError("gdn_fused needs the Gated-DeltaNet write (u, w None)")
    o = np.zeros((B, T, H, dv))
    Sf = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dv, dk)) if S0 is None else S0[b, h].copy()
            for c0 in range(0, T, chunk):
                c1 = min(T, c0 + chunk)
                Kc, Qc = k[b, c0:c1, h], q[b, c0:c1, h]
                ac, bc = alpha[b, c0:c1, h], beta[b, c0:c1, h]
                Uc, Wc = u[b, c0:c1, h], w[b, c0:c1, h]
                tm = chunk_terms(Kc, Qc, ac, bc, Uc, Wc)
                gam, D = tm["gam"], tm["D"]
                if gdn_fused:
                    Vc = v[b, c0:c1, h]
                    Ups = tm["T"] @ (bc[:, None] * Vc)
                    Y = Ups - tm["Wk"] @ S.T
                    o[b, c0:c1, h] = gam[:, None] * (Qc @ S.T) + tm["Mqk"] @ Y
                    S = gam[-1] * S + Y.T @ (D[:, None] * Kc)
                else:
                    X = tm["Wk"] @ S.T + tm["Xu"]
                    o[b, c0:c1, h] = (gam[:, None] * (Qc @ S.T) - tm["Mqk"] @ X
                                      + tm["Mqw"] @ tm["Ut"])
                    S = (gam[-1] * S - X.T @ (D[:, None] * Kc)
                         + tm["Ut"].T @ (tm["Dt"][:, None] * tm["Wt"]))
            Sf[b, h] = S
    return o, Sf
