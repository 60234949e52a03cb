"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each pin follows from the definition of the scan (PRISM, gist.science explainer, technical summary
2.1 and 2.2; banbantang.com PRISM article, section 1(4)) or from the affine-monoid view of
"Sequential Parallel Duality in Prefix Scannable Models" (papernotes, key design 2: the element
(E_t, f_t), its associative composition with identity (I, 0), and the Blelloch scan).  The last
test plants known mistakes in the oracle and checks that some pin catches every one.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from delta_rule_sequence_b200.workloads import WORKLOADS, make_inputs
from tests.chunk_algebra import chunk_element, chunk_terms, chunked_forward

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------------------------
# small input builders (fp32 so that every value is exact in the oracle's double arithmetic)

def _rand_case(seed, B=2, T=13, H=2, dk=6, dv=5, L=3, gdn=False, s0=True, dyadic=False):
    g = torch.Generator().manual_seed(seed)
    def rn(*shape):
        x = torch.randn(shape, generator=g)
        if dyadic:  # few mantissa bits: sums and products below stay exact in fp32
            x = torch.round(x * 8) / 8
        return x.float()
    q = rn(B, T, H, dk)
    k = torch.nn.functional.normalize(torch.randn((B, T, H, dk), generator=g), dim=-1).float()
    alpha = torch.exp(-torch.nn.functional.softplus(torch.randn((B, T, H), generator=g) - 1)).float()
    beta = torch.sigmoid(torch.randn((B, T, H), generator=g)).float()
    v = rn(B, T, H, dv)
    u = w = None
    if not gdn:
        u = rn(B, T, H, L, dv)
        w = torch.nn.functional.normalize(torch.randn((B, T, H, L, dk), generator=g), dim=-1).float()
    S0 = rn(B, H, dv, dk) * 0.5 if s0 else None
    return dict(q=q, k=k, v=v, alpha=alpha, beta=beta, u=u, w=w, S0=S0)


def _np(x):
    return None if x is None else x.double().numpy()


# ----------------------------------------------------------------------------------------------
# pin 1: brute-force Blelloch scan over explicit affine elements (associativity + element form)

def _elements(x, b, h):
    """E_t = alpha_t (I - beta_t k_t k_t^T), f_t = sum_l u_{t,l} w_{t,l}^T, so S_t = S_{t-1}E_t+f_t."""
    k = _np(x["k"])[b, :, h]
    T, dk = k.shape
    a = _np(x["alpha"])[b, :, h]
    be = _np(x["beta"])[b, :, h]
    if x["u"] is None:
        u = (be[:, None] * _np(x["v"])[b, :, h])[:, None, :]
        w = k[:, None, :]
    else:
        u = _np(x["u"])[b, :, h]
        w = _np(x["w"])[b, :, h]
    els = []
    for t in range(T):
        E = a[t] * (np.eye(dk) - be[t] * np.outer(k[t], k[t]))
        f = sum(np.outer(u[t, l], w[t, l]) for l in range(u.shape[1]))
        els.append((E, f))
    return els


def _compose(x, y):
    """x applied first, then y: S -> (S E_x + f_x) E_y + f_y."""
    return (x[0] @ y[0], x[1] @ y[0] + y[1])


def _blelloch_exclusive(els, dk, dv):
    n = 1
    while n < len(els):
        n *= 2
    ident = (np.eye(dk), np.zeros((dv, dk)))
    a = list(els) + [ident] * (n - len(els))
    d = 1
    while d < n:                                   # up-sweep
        for i in range(0, n, 2 * d):
            a[i + 2 * d - 1] = _compose(a[i + d - 1], a[i + 2 * d - 1])
        d *= 2
    a[n - 1] = ident
    d = n // 2
    while d >= 1:                                  # down-sweep
        for i in range(0, n, 2 * d):
            left = a[i + d - 1]
            a[i + d - 1] = a[i + 2 * d - 1]
            a[i + 2 * d - 1] = _compose(a[i + 2 * d - 1], left)
        d //= 2
    return a[:len(els)]


def pin_blelloch(x, run):
    o, Sf = run(x)
    B, T, H, dk = x["q"].shape
    err = 0.0
    for b in range(B):
        for h in range(H):
            els = _elements(x, b, h)
            dv = els[0][1].shape[0]
            excl = _blelloch_exclusive(els, dk, dv)
            S0 = np.zeros((dv, dk)) if x["S0"] is None else _np(x["S0"])[b, h]
            q = _np(x["q"])[b, :, h]
            for t in range(T):
                E, f = _compose(excl[t], els[t])
                St = S0 @ E + f
                err = max(err, np.abs(St @ q[t] - o[b, t, h]).max())
            err = max(err, np.abs(St - Sf[b, h]).max())
    return err


@pytest.mark.parametrize("gdn", [False, True])
def test_blelloch_matches_oracle(gdn):
    x = _rand_case(1, T=13, gdn=gdn)
    assert pin_blelloch(x, lambda x: oracle.scan_ref(**x)) < 1e-12


def test_composition_is_associative_with_identity():
    x = _rand_case(2, T=3)
    e = _elements(x, 0, 0)
    lhs = _compose(_compose(e[0], e[1]), e[2])
    rhs = _compose(e[0], _compose(e[1], e[2]))
    assert np.abs(lhs[0] - rhs[0]).max() < 1e-14 and np.abs(lhs[1] - rhs[1]).max() < 1e-14
    ident = (np.eye(6), np.zeros((5, 6)))
    for z in (_compose(ident, e[0]), _compose(e[0], ident)):
        assert np.abs(z[0] - e[0][0]).max() == 0 and np.abs(z[1] - e[0][1]).max() == 0


# ----------------------------------------------------------------------------------------------
# pin 2: causal linear attention closed form (alpha = 1, beta = 0, u = v, w = k, S0 = 0)

def pin_linear_attention(run):
    x = _rand_case(3, T=17, L=1, s0=False)
    x["alpha"][:] = 1.0
    x["beta"][:] = 0.0
    x["u"] = x["v"][:, :, :, None, :].clone()
    x["w"] = x["k"][:, :, :, None, :].clone()
    o, Sf = run(x)
    q, k, v = _np(x["q"]), _np(x["k"]), _np(x["v"])
    err = 0.0
    for b in range(q.shape[0]):
        for h in range(q.shape[2]):
            Q, K, V = q[b, :, h], k[b, :, h], v[b, :, h]
            o_ref = np.tril(Q @ K.T) @ V                     # o_t = sum_{s<=t} v_s (k_s . q_t)
            err = max(err, np.abs(o_ref - o[b, :, h]).max(), np.abs(V.T @ K - Sf[b, h]).max())
    return err


def test_linear_attention_closed_form():
    assert pin_linear_attention(lambda x: oracle.scan_ref(**x)) < 1e-12


# ----------------------------------------------------------------------------------------------
# pin 3: gated linear attention closed form (beta = 0): pure decay plus rank-L writes

def pin_gated_linear_attention(run):
    x = _rand_case(4, T=19, L=3)
    x["beta"][:] = 0.0
    o, Sf = run(x)
    q, a, u, w, S0 = (_np(x[n]) for n in ("q", "alpha", "u", "w", "S0"))
    err = 0.0
    B, T, H, dk = q.shape
    for b in range(B):
        for h in range(H):
            g = np.cumsum(np.log(a[b, :, h]))
            for t in range(T):
                ref = np.exp(g[t]) * S0[b, h] @ q[b, t, h]
                for s in range(t + 1):
                    ref = ref + np.exp(g[t] - g[s]) * (u[b, s, h] .T @ (w[b, s, h] @ q[b, t, h]))
                err = max(err, np.abs(ref - o[b, t, h]).max())
            Sref = np.exp(g[-1]) * S0[b, h]
            for s in range(T):
                Sref = Sref + np.exp(g[-1] - g[s]) * (u[b, s, h].T @ w[b, s, h])
            err = max(err, np.abs(Sref - Sf[b, h]).max())
    return err


def test_gated_linear_attention_closed_form():
    assert pin_gated_linear_attention(lambda x: oracle.scan_ref(**x)) < 1e-12


# ----------------------------------------------------------------------------------------------
# pin 4: the delta-rule overwrite.  With |k_t| = 1 exactly:
#   S_t k_t = alpha_t (1 - beta_t) S_{t-1} k_t + sum_l u_{t,l} (w_{t,l} . k_t)
# and with alpha = beta = 1 and the GDN write, reading with q_t = k_t returns v_t exactly.

def _exact_unit_keys(g, B, T, H, dk):
    """Keys with four entries of +-1/2 and the rest zero: unit norm exactly in binary."""
    k = torch.zeros((B, T, H, dk))
    for idx in np.ndindex(B, T, H):
        pos = torch.randperm(dk, generator=g)[:4]
        sgn = torch.randint(0, 2, (4,), generator=g).float() * 2 - 1
        k[idx][pos] = 0.5 * sgn
    return k


def pin_overwrite(run):
    g = torch.Generator().manual_seed(5)
    x = _rand_case(5, T=11, dk=8, dv=6, L=2)
    x["k"] = _exact_unit_keys(g, 2, 11, 2, 8)
    x["q"] = x["k"].clone()
    err = 0.0
    o, Sf = run(x)
    # general identity at every t >= 1, using the oracle's own state after t-1 tokens
    for t in range(1, 11):
        xp = {n: (None if v is None else v[:, :t].contiguous() if n not in ("S0",) else v)
              for n, v in x.items()}
        _, S_prev = run(xp)
        kt = _np(x["k"])[:, t]
        a, be = _np(x["alpha"])[:, t], _np(x["beta"])[:, t]
        u, w = _np(x["u"])[:, t], _np(x["w"])[:, t]
        for b in range(2):
            for h in range(2):
                lhs = o[b, t, h]  # q_t = k_t, so o_t = S_t k_t
                rhs = a[b, h] * (1 - be[b, h]) * (S_prev[b, h] @ kt[b, h])
                rhs = rhs + u[b, h].T @ (w[b, h] @ kt[b, h])
                err = max(err, np.abs(lhs - rhs).max())
    # full overwrite with the GDN write
    y = _rand_case(6, T=9, dk=8, dv=6, gdn=True)
    y["k"] = _exact_unit_keys(g, 2, 9, 2, 8)
    y["q"] = y["k"].clone()
    y["alpha"][:] = 1.0
    y["beta"][:] = 1.0
    o2, _ = run(y)
    err = max(err, np.abs(o2 - _np(y["v"])).max())
    return err


def test_delta_overwrite_identity():
    assert pin_overwrite(lambda x: oracle.scan_ref(**x)) < 1e-12


# ----------------------------------------------------------------------------------------------
# pin 5: superposition (jointly linear in S0 and u) and row independence

def pin_superposition(run):
    xa = _rand_case(7, T=10, dyadic=True)
    xb = _rand_case(8, T=10, dyadic=True)
    for n in ("q", "k", "alpha", "beta", "w", "v"):
        xb[n] = xa[n]
    xs = dict(xa)
    xs["u"] = xa["u"] + xb["u"]          # exact: dyadic values with few mantissa bits
    xs["S0"] = xa["S0"] + xb["S0"]
    oa, Sa = run(xa)
    ob, Sb = run(xb)
    os_, Ss = run(xs)
    err = max(np.abs(oa + ob - os_).max(), np.abs(Sa + Sb - Ss).max())
    # row independence: permuting value rows of (S0, u) permutes rows of (o, S_final)
    perm = torch.tensor([3, 0, 4, 1, 2])
    xp = dict(xa)
    xp["u"] = xa["u"][..., perm].contiguous()
    xp["S0"] = xa["S0"][:, :, perm].contiguous()
    op, Sp = run(xp)
    err = max(err, np.abs(op - oa[..., perm.numpy()]).max(),
              np.abs(Sp - Sa[:, :, perm.numpy()]).max())
    return err


def test_superposition_and_row_independence():
    assert pin_superposition(lambda x: oracle.scan_ref(**x)) < 1e-12


# ----------------------------------------------------------------------------------------------
# pin 6: resumability -- S_final of a prefix is the entry state of the rest

@pytest.mark.parametrize("T1", [1, 6, 12])
def test_resumable_split(T1):
    x = _rand_case(9, T=13)
    o, Sf = oracle.scan_ref(**x)
    first = {n: (v if v is None or n == "S0" else v[:, :T1].contiguous()) for n, v in x.items()}
    rest = {n: (v if v is None or n == "S0" else v[:, T1:].contiguous()) for n, v in x.items()}
    o1, S1 = oracle.scan_ref(**first)
    rest["S0"] = torch.from_numpy(S1)
    o2, S2 = oracle.scan_ref(**rest)
    assert np.abs(np.concatenate([o1, o2], axis=1) - o).max() < 1e-13
    assert np.abs(S2 - Sf).max() < 1e-13


# ----------------------------------------------------------------------------------------------
# pin 7: the Gated-DeltaNet route equals the general route with u = beta v, w = k (L = 1)

def pin_gdn_route(run):
    x = _rand_case(10, T=12, gdn=True, dyadic=True)
    x["beta"] = torch.round(x["beta"] * 8) / 8        # beta * v exact in fp32
    og, Sg = run(x)
    y = dict(x)
    y["u"] = (x["beta"][..., None] * x["v"])[:, :, :, None, :].contiguous()
    y["w"] = x["k"][:, :, :, None, :].contiguous()
    ou, Su = run(y)
    return max(np.abs(og - ou).max(), np.abs(Sg - Su).max())


def test_gdn_route_equals_general_route():
    assert pin_gdn_route(lambda x: oracle.scan_ref(**x)) < 1e-13


# ----------------------------------------------------------------------------------------------
# pin 8: a two-step example worked by hand in exact arithmetic

def pin_hand_worked(run):
    with open(os.path.join(GOLDEN, "hand_worked_gdn_d2.json")) as f:
        gd = json.load(f)
    t = lambda a: torch.tensor(a, dtype=torch.float32)
    x = dict(q=t(gd["q"])[None, :, None], k=t(gd["k"])[None, :, None],
             v=t(gd["v"])[None, :, None], alpha=t(gd["alpha"])[None, :, None],
             beta=t(gd["beta"])[None, :, None], u=None, w=None,
             S0=t(gd["S0"])[None, None])
    o, Sf = run(x)
    return max(np.abs(o[0, :, 0] - np.array(gd["o"])).max(),
               np.abs(Sf[0, 0] - np.array(gd["S_final"])).max())


def test_hand_worked_example():
    assert pin_hand_worked(lambda x: oracle.scan_ref(**x)) == 0.0


# ----------------------------------------------------------------------------------------------
# the chunked (UT-transform) algebra that the kernels implement equals the recurrence

@pytest.mark.parametrize("chunk", [1, 2, 4, 8, 16, 64, 128])
def test_chunked_algebra_matches_oracle(chunk):
    x = _rand_case(11, T=150, dk=8, dv=6, L=3)
    o, Sf = oracle.scan_ref(**x)
    oc, Sc = chunked_forward(**x, chunk=chunk)
    assert np.abs(oc - o).max() < 1e-9 * (1 + np.abs(o).max())
    assert np.abs(Sc - Sf).max() < 1e-9 * (1 + np.abs(Sf).max())


@pytest.mark.parametrize("chunk", [4, 64])
def test_chunked_gdn_fused_algebra_matches_oracle(chunk):
    x = _rand_case(12, T=130, dk=8, dv=6, gdn=True)
    o, Sf = oracle.scan_ref(**x)
    oc, Sc = chunked_forward(**x, chunk=chunk, gdn_fused=True)
    assert np.abs(oc - o).max() < 1e-9 * (1 + np.abs(o).max())
    assert np.abs(Sc - Sf).max() < 1e-9 * (1 + np.abs(Sf).max())


def test_chunk_affine_element_and_segment_composition():
    """S' = S E_c + f_c per chunk, and composing chunk elements gives a segment element."""
    x = _rand_case(13, B=1, H=1, T=24, dk=5, dv=4, L=2)
    k, q, a, be = (_np(x[n])[0, :, 0] for n in ("k", "q", "alpha", "beta"))
    u, w = _np(x["u"])[0, :, 0], _np(x["w"])[0, :, 0]
    seg = (np.eye(5), np.zeros((4, 5)))
    for c0 in range(0, 24, 8):
        tm = chunk_terms(k[c0:c0 + 8], q[c0:c0 + 8], a[c0:c0 + 8], be[c0:c0 + 8],
                         u[c0:c0 + 8], w[c0:c0 + 8])
        seg = _compose(seg, chunk_element(k[c0:c0 + 8], tm, 4))
    _, Sf = oracle.scan_ref(**x)
    S0 = _np(x["S0"])[0, 0]
    assert np.abs(S0 @ seg[0] + seg[1] - Sf[0, 0]).max() < 1e-12


def test_workload_shapes_scale_to_oracle():
    """Every named workload runs through the oracle at a reduced length."""
    for name, wl in WORKLOADS.items():
        small = wl.with_(B=min(wl.B, 2), H=min(wl.H, 2), T=min(max(wl.T, 1), 20))
        x = make_inputs(small)
        o, Sf = oracle.scan_ref(**x)
        assert np.isfinite(o).all() and np.isfinite(Sf).all()
        assert o.shape == (small.B, small.T, small.H, small.dv)


# ----------------------------------------------------------------------------------------------
# planted mistakes: every mutant of the oracle fails at least one pin

PINS = {
    "blelloch_general": lambda run: pin_blelloch(_rand_case(1, T=13), run),
    "blelloch_gdn": lambda run: pin_blelloch(_rand_case(1, T=13, gdn=True), run),
    "blelloch_square": lambda run: pin_blelloch(_rand_case(14, T=9, dk=5, dv=5), run),
    "linear_attention": pin_linear_attention,
    "gated_linear_attention": pin_gated_linear_attention,
    "overwrite": pin_overwrite,
    "hand_worked": pin_hand_worked,
    "gdn_route": pin_gdn_route,
}


@pytest.mark.parametrize("mutation", [1, 2, 3, 4, 5, 6, 7])
def test_pins_catch_planted_mistakes(mutation):
    run = lambda x: oracle.scan_ref(**x, mutation=mutation)
    caught = [name for name, pin in PINS.items() if pin(run) > 1e-6]
    assert caught, f"mutation {mutation} passed every pin"
