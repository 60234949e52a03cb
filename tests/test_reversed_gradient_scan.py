"""CPU checks of the chunk-parallel backward's gradient scan (csrc/scan_bwd.cu), in fp64 numpy.

The backward runs the gradient of the state, G_t (after token t), as the forward scan's own
recurrence over the reversed tokens: G_{t-1} = G_t A_t + dO_{t-1} q_{t-1}^T with
A_t = alpha_t (I - beta_t k_t k_t^T), P = C - T mod C identity positions in front (the last of them
writing dO_{T-1} q_{T-1}^T onto the entry state dS_final), a checkpoint of the state at every
C-token chunk start, and the exit state dS0.  The gradient at the end of forward chunk c, excluding
that chunk's own outputs, is then the checkpoint NR - 1 - c less dO q^T of the chunk's last token.
These tests lay the reversed sequence out the way the kernel does and check dS0 against the
backward oracle (oracle/scan_grad.py) and every chunk-end gradient against the direct reverse
recurrence, for T around the chunk length."""
import numpy as np
import pytest

from oracle.scan_grad import scan_grad_ref


def _inputs(T, d, seed):
    g = np.random.default_rng(seed)
    k = g.normal(size=(T, d))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    return dict(q=g.normal(size=(T, d)), k=k, alpha=g.uniform(0.7, 1.0, T), beta=g.uniform(0.0, 1.0, T),
                do=g.normal(size=(T, d)), dSf=g.normal(size=(d, d)), v=g.normal(size=(T, d)))


def _reversed_layout(T, C):
    """(transition token, write token) of every position of the gradient scan, as the kernel builds
    them (-1 = none), and P, NR."""
    P = C - T % C
    pos = []
    for p in range(T + P):
        if p < P:
            pos.append((-1, T - 1 if p == P - 1 else -1))
        else:
            tk = T - 1 - (p - P)
            pos.append((tk, tk - 1))
    return pos, P, (T + P) // C


def _gradient_scan(x, T, C):
    d = x["q"].shape[1]
    A = [x["alpha"][t] * (np.eye(d) - x["beta"][t] * np.outer(x["k"][t], x["k"][t])) for t in range(T)]
    pos, P, NR = _reversed_layout(T, C)
    S, ck = x["dSf"].copy(), []
    for p, (tk, tw) in enumerate(pos):
        if p % C == 0:
            ck.append(S.copy())
        if tk >= 0:
            S = S @ A[tk]
        if tw >= 0:
            S = S + np.outer(x["do"][tw], x["q"][tw])
    return S, ck, A, NR


@pytest.mark.parametrize("T", [1, 2, 7, 8, 9, 15, 16, 17, 24, 31])
def test_gradient_scan_exit_state_is_dS0(T):
    C = 8
    x = _inputs(T, 4, seed=T)
    dS0, _, _, _ = _gradient_scan(x, T, C)
    r = lambda a: a[None, :, None]  # [T, ...] -> [1, T, 1, ...]
    ref = scan_grad_ref(r(x["q"]), r(x["k"]), r(x["v"]), x["alpha"][None, :, None], x["beta"][None, :, None],
                        do=r(x["do"]), dS_final=x["dSf"][None, None])
    np.testing.assert_allclose(dS0, ref["dS0"][0, 0], rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("T", [1, 5, 8, 9, 16, 23, 24, 25])
def test_gradient_scan_checkpoints_give_every_chunk_end_gradient(T):
    C = 8
    x = _inputs(T, 4, seed=100 + T)
    _, ck, A, NR = _gradient_scan(x, T, C)
    # the direct reverse recurrence: G[t] includes token t's own output term
    G = [None] * T
    G[T - 1] = x["dSf"] + np.outer(x["do"][T - 1], x["q"][T - 1])
    for t in range(T - 2, -1, -1):
        G[t] = G[t + 1] @ A[t + 1] + np.outer(x["do"][t], x["q"][t])
    nch = (T + C - 1) // C
    assert NR in (nch, nch + 1)
    for c in range(nch):
        g = ck[NR - 1 - c].copy()
        tl = (c + 1) * C - 1  # the chunk's last token
        if tl < T:
            g -= np.outer(x["do"][tl], x["q"][tl])
        # the gradient at the chunk's end from the tokens after it (dS_final for the last chunk)
        want = x["dSf"] if tl >= T - 1 else G[tl + 1] @ A[tl + 1]
        np.testing.assert_allclose(g, want, rtol=1e-10, atol=1e-10)
