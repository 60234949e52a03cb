"""fp64 oracle for the input-anchored write-term producer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import this module.  It shares no code with the CUDA library and imports
nothing from it.

What it computes, per (batch b, head h) and token t, after "PRISM: Parallel Residual Iterative
Sequence Model" (gist.science explainer), technical summary section 2.2 (input-anchored loop
unrolling), with the ShortConv width from the banbantang.com PRISM article, section 5(1) (the
anchor covers the last 3-4 tokens) and the first residual from its section 3(4) (at the first step
the residual is the input itself):

    anchor       a_t = sum_{j=0..3} c_j * x_{t-j}            (depthwise, causal; x_{<0} = 0)
    directions   k_t^(l) = W_k^(l) a_t,   gains  p_t^(l) = W_p^(l) a_t          l = 1..L
    residual     r_t^(1) = v_t,   delta_t^(l) = GELU(p_t^(l) * r_t^(l)),   r_t^(l+1) = r_t^(l) - delta_t^(l)
    write terms  u_{t,l} = beta_t^(l) delta_t^(l),   w_{t,l} = k_t^(l)

so that the scan's write sum_l u_{t,l} w_{t,l}^T is the summary's B_t = sum_l beta delta k^T.
GELU is the exact one, x Phi(x) with Phi the standard normal CDF (math.erf).

The loops follow the definition step by step (one token, one rank, one element at a time for the
nonlinear chain); a matrix-vector product is numpy's.  Pins: ``tests/test_producer_pins.py``.
"""
from __future__ import annotations

import math

import numpy as np

CONV_WIDTH = 4


def _f64(a):
    """A torch tensor (any dtype, bf16 included) or array as float64 numpy."""
    if hasattr(a, "detach"):
        return a.detach().to("cpu").double().numpy()
    return np.asarray(a, dtype=np.float64)


def gelu(x: float) -> float:
    return 0.5 * x * (1.0 + math.erf(x / math.sqrt(2.0)))


def write_producer_ref(x, v, conv, Wk, Wp, beta, *, mutant: int = 0):
    """x, v: [B,T,H,d]; conv: [H,4,d] (c_0 multiplies x_t); Wk, Wp: [H,L,d,d] (row = output
    index); beta: [B,T,H,L].  Returns (u [B,T,H,L,d], w [B,T,H,L,d], r_final [B,T,H,d]) in fp64.

    ``mutant`` plants one mistake, for the pin tests only: 1 the convolution reads x_{t+j}
    (not causal); 2 the tanh approximation of GELU; 3 the residual is never updated; 4 W_k is
    applied transposed; 5 beta gates the residual update as well; 6 the anchor drops its c_0 term.
    """
    x, v, conv, Wk, Wp, beta = (_f64(t) for t in (x, v, conv, Wk, Wp, beta))
    B, T, H, d = x.shape
    L = Wk.shape[1]
    u = np.zeros((B, T, H, L, d))
    w = np.zeros((B, T, H, L, d))
    r_final = np.zeros((B, T, H, d))

    def act(z):
        if mutant == 2:
            return 0.5 * z * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (z + 0.044715 * z ** 3)))
        return gelu(z)

    for b in range(B):
        for h in range(H):
            for t in range(T):
                a = np.zeros(d)
                for j in range(CONV_WIDTH):
                    if mutant == 6 and j == 0:
                        continue
                    s = t + j if mutant == 1 else t - j
                    if 0 <= s < T:
                        a += conv[h, j] * x[b, s, h]
                r = v[b, t, h].copy()
                for l in range(L):
                    k_l = (Wk[h, l].T if mutant == 4 else Wk[h, l]) @ a
                    p_l = Wp[h, l] @ a
                    delta = np.array([act(p_l[i] * r[i]) for i in range(d)])
                    u[b, t, h, l] = beta[b, t, h, l] * delta
                    w[b, t, h, l] = k_l
                    if mutant == 3:
                        continue
                    r = r - (beta[b, t, h, l] * delta if mutant == 5 else delta)
                r_final[b, t, h] = r
    return u, w, r_final
