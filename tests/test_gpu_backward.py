"""GPU parity of the backward pass (prism_scan_bwd, through the C ABI) against the fp64 backward
oracle (oracle/scan_grad.py, itself pinned by finite differences of the forward oracle), element by
element on the same seeded bytes: every gradient (dq, dk, dv or du and dw, dalpha, dbeta, dS0) for
both write forms, bf16 and fp32 I/O, widths 32/64/128 and dk != dv, ragged T around the 64-token
checkpoint interval, T = 0, edge regimes, and sampled heads of the full-size gdn workload and of
the long-context one over its first 4096 tokens.
Tolerance: |x - r| <= tol (1 + |r|), tol = 2e-2 for bf16 I/O, 1e-4 for fp32 I/O."""
import numpy as np
import pytest
import torch

from oracle.scan_grad import scan_grad_ref
from delta_rule_sequence_b200.workloads import WORKLOADS, make_inputs, select_heads
from tests.parity import TOL, compare, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from delta_rule_sequence_b200 import build

    build.build()


def _upstream(wl, seed, with_dS=True):
    """Seeded upstream gradients: dO ~ N(0, 1) in the I/O type, dS_final ~ N(0, 0.1^2) fp32."""
    g = torch.Generator().manual_seed(5000 + seed)
    dO = torch.randn((wl.B, wl.T, wl.H, wl.dv), generator=g).to(wl.torch_io)
    dS = (torch.randn((wl.B, wl.H, wl.dv, wl.dk), generator=g) * 0.1).float() if with_dS else None
    return dO, dS


def _run(x, dO, dS):
    from delta_rule_sequence_b200.prism import prism_scan_bwd

    d = to_device(x)
    out = prism_scan_bwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["u"], d["w"], d["S0"],
                         dO=dO.cuda(), dS_final=None if dS is None else dS.cuda())
    torch.cuda.synchronize()
    return {n: (None if t is None else t.cpu().numpy()) for n, t in out.items()}


def _check(got, ref, tol, names):
    for n in names:
        compare(n, got[n], ref[n], tol)


def _names(gdn, dS0=True):
    base = ["dq", "dk", "dalpha", "dbeta"] + (["dv"] if gdn else ["du", "dw"])
    return base + (["dS0"] if dS0 else [])


@pytest.mark.parametrize("name,over", [
    ("gdn", dict(B=1, H=2, T=200)),
    ("gdn", dict(B=2, H=1, T=64, dk=64, dv=64)),
    ("tiny", dict(T=150)),
    ("recsys", dict(B=1, H=2, T=130, L=3)),
    ("long", dict(H=2, T=77, chunk=64)),
    ("recsys", dict(B=1, H=2, T=100, L=2, io="f32")),
    ("recsys", dict(B=1, H=1, T=90, dk=32, dv=64, L=2, io="f32")),
    ("gdn", dict(B=1, H=2, T=129, dk=128, dv=64, io="f32")),
    # chunk-parallel form at its edges: one token, and one token past a chunk
    ("gdn", dict(B=1, H=2, T=1)),
    ("recsys", dict(B=1, H=1, T=65, L=2)),
])
def test_backward_matches_oracle(name, over):
    wl = WORKLOADS[name].with_(**over)
    x = make_inputs(wl, seed=wl.T)
    dO, dS = _upstream(wl, wl.T)
    got = _run(x, dO, dS)
    ref = scan_grad_ref(**x, do=dO, dS_final=dS)
    _check(got, ref, TOL[wl.io], _names(x["u"] is None))


def test_backward_without_state_gradient_and_without_S0():
    wl = WORKLOADS["long"].with_(H=2, T=100, chunk=64, s0_std=0.0)
    x = make_inputs(wl, seed=3)
    dO, _ = _upstream(wl, 3, with_dS=False)
    got = _run(x, dO, None)
    ref = scan_grad_ref(**x, do=dO, dS_final=None)
    _check(got, ref, TOL["bf16"], _names(False))


def test_backward_no_tokens_passes_the_state_gradient_through():
    from delta_rule_sequence_b200.prism import prism_scan_bwd

    wl = WORKLOADS["long"].with_(H=2, T=1, chunk=64)
    x = to_device(make_inputs(wl))
    dS = torch.randn((1, 2, 128, 128), device="cuda")
    cut = lambda t: t[:, :0].contiguous()
    out = prism_scan_bwd(cut(x["q"]), cut(x["k"]), None, cut(x["alpha"]), cut(x["beta"]),
                         cut(x["u"]), cut(x["w"]), x["S0"], dO=cut(x["q"]), dS_final=dS)
    torch.cuda.synchronize()
    assert torch.equal(out["dS0"], dS)


def test_backward_edge_regimes():
    """Strong decay, beta = 1 and no decay with no erase (the state only grows), rank-L write."""
    wl = WORKLOADS["recsys"].with_(B=1, H=2, T=150, L=2)
    for case in ("strong_decay", "beta_one", "linear"):
        x = make_inputs(wl, seed=9)
        g = torch.Generator().manual_seed(9)
        if case == "strong_decay":
            x["alpha"] = (0.01 + 0.19 * torch.rand((1, 150, 2), generator=g)).float()
        elif case == "beta_one":
            x["beta"][:] = 1.0
        else:
            x["alpha"][:] = 1.0
            x["beta"][:] = 0.0
        dO, dS = _upstream(wl, 9)
        got = _run(x, dO, dS)
        ref = scan_grad_ref(**x, do=dO, dS_final=dS)
        _check(got, ref, TOL["bf16"], _names(False))


@pytest.mark.parametrize("name,over,heads", [("gdn", {}, [(0, 0), (3, 7)]),
                                             ("long", dict(T=4096), [(0, 11)])])
def test_backward_full_size_sampled(name, over, heads):
    """The gdn workload at full size (and the long-context one over its first 4096 tokens: the
    oracle keeps every state of a sequence) in one launch; the listed (b, h) sequences against the
    oracle."""
    wl = WORKLOADS[name].with_(**over)
    x = make_inputs(wl)
    dO, dS = _upstream(wl, 1)
    got = _run(x, dO, dS)
    sub = select_heads(x, heads)
    dO_s = torch.cat([dO[b:b + 1, :, h:h + 1] for b, h in heads], 0)
    dS_s = torch.cat([dS[b:b + 1, h:h + 1] for b, h in heads], 0)
    ref = scan_grad_ref(**sub, do=dO_s, dS_final=dS_s)
    gdn = x["u"] is None
    for n in _names(gdn):
        if n == "dS0":
            g = np.concatenate([got[n][b:b + 1, h:h + 1] for b, h in heads], 0)
        else:
            g = np.concatenate([got[n][b:b + 1, :, h:h + 1] for b, h in heads], 0)
        compare(n, g, ref[n], TOL[wl.io])
