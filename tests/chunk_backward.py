"""fp64 numpy mirror of a chunked backward pass, the design a GPU backward would follow.

Test helper, not the oracle.  Per head, with chunk-entry states S_c and the chunk element
(E_c, f_c) (S_{c+1} = S_c E_c + f_c, tests/chunk_algebra.py), the outputs of chunk c split as
O_c = Qt_c S_c^T + (terms of the chunk's own tokens) with Qt_c = diag(gamma) Q - Mqk Wk, so the
gradient of the loss with respect to a chunk-entry state obeys the reverse chunk recurrence

    dS_C = dS_final,      dS_c = dS_{c+1} E_c^T + dO_c^T Qt_c

(in order over chunks, like the forward's state pass), and given S_c and dS_{c+1}, every chunk's
input gradients follow from the token-level backward run on that chunk alone (all chunks at
once).  ``chunked_backward`` assembles the gradients this way, taking the per-chunk token-level
step from the backward oracle; tests/test_chunk_backward.py checks it against the backward oracle
on the whole sequence.
"""
from __future__ import annotations

import numpy as np

from oracle.scan_grad import scan_grad_ref
from tests.chunk_algebra import _to64, chunk_element, chunk_terms


def chunked_backward(q, k, v, alpha, beta, u=None, w=None, S0=None, *, do, dS_final=None, chunk=64):
    q, k, v, alpha, beta, do = map(_to64, (q, k, v, alpha, beta, do))
    u, w, S0, dS_final = _to64(u), _to64(w), _to64(S0), _to64(dS_final)
    B, T, H, dk = q.shape
    gdn = u is None
    dv = v.shape[3] if gdn else u.shape[4]
    # the chunk algebra works on the general write: u = beta v, w = k for the GDN write
    ug = (beta[..., None] * v)[:, :, :, None, :] if gdn else u
    wg = k[:, :, :, None, :] if gdn else w
    grads = {n: None for n in ("dq", "dk", "dv", "dalpha", "dbeta", "du", "dw")}
    grads.update(dq=np.zeros_like(q), dk=np.zeros_like(k), dalpha=np.zeros_like(alpha),
                 dbeta=np.zeros_like(beta), dS0=np.zeros((B, H, dv, dk)), dS_entry=[])
    if gdn:
        grads["dv"] = np.zeros_like(v)
    else:
        grads["du"], grads["dw"] = np.zeros_like(u), np.zeros_like(w)
    bounds = [(c0, min(T, c0 + chunk)) for c0 in range(0, T, chunk)]
    for b in range(B):
        for h in range(H):
            # forward: chunk-entry states and the per-chunk terms
            S = np.zeros((dv, dk)) if S0 is None else S0[b, h].copy()
            entry, elems, qts = [], [], []
            for c0, c1 in bounds:
                tm = chunk_terms(k[b, c0:c1, h], q[b, c0:c1, h], alpha[b, c0:c1, h],
                                 beta[b, c0:c1, h], ug[b, c0:c1, h], wg[b, c0:c1, h])
                E, f = chunk_element(k[b, c0:c1, h], tm, dv)
                entry.append(S)
                elems.append(E)
                qts.append(tm["gam"][:, None] * q[b, c0:c1, h] - tm["Mqk"] @ tm["Wk"])
                S = S @ E + f
            # reverse chunk recurrence for the state gradients at chunk boundaries
            dS = np.zeros((dv, dk)) if dS_final is None else dS_final[b, h].copy()
            exit_grad = [None] * len(bounds)
            for c in reversed(range(len(bounds))):
                c0, c1 = bounds[c]
                exit_grad[c] = dS
                dS = dS @ elems[c].T + do[b, c0:c1, h].T @ qts[c]
            grads["dS0"][b, h] = dS
            grads["dS_entry"].append(dS)
            # every chunk's own gradients, independently of the others
            for c, (c0, c1) in enumerate(bounds):
                sl = lambda x: None if x is None else x[b:b + 1, c0:c1, h:h + 1]
                g = scan_grad_ref(sl(q), sl(k), sl(v), sl(alpha), sl(beta), sl(u), sl(w),
                                  entry[c][None, None], do=sl(do), dS_final=exit_grad[c][None, None])
                for n in ("dq", "dk", "dalpha", "dbeta") + (("dv",) if gdn else ("du", "dw")):
                    grads[n][b, c0:c1, h] = g[n][0, :, 0]
    return grads
