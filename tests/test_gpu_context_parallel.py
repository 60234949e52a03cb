"""GPU parity of the context-parallel building blocks: the segment element (E, f) of
prism_scan_segment_element, the fold prism_state_fold, and a two-segment scan run the way two ranks
would run it (element of segment 1, fold, forward of segment 2), all against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from delta_rule_sequence_b200.workloads import WORKLOADS, make_inputs
from tests.parity import TOL, compare, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from delta_rule_sequence_b200 import build

    build.build()


def _oracle_element(x):
    """E from S0 = I with the write switched off, f from S0 = 0 with the write."""
    B, T, H, dk = x["q"].shape
    eye = np.broadcast_to(np.eye(dk), (B, H, dk, dk)).copy()
    if x["u"] is None:
        _, E = oracle.scan_ref(x["q"], x["k"], torch.zeros_like(x["v"]), x["alpha"], x["beta"], S0=eye)
    else:
        _, E = oracle.scan_ref(x["q"], x["k"], None, x["alpha"], x["beta"], torch.zeros_like(x["u"]),
                               x["w"], S0=eye)
    _, f = oracle.scan_ref(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["u"], x["w"], None)
    return E, f


ELEMENT_CASES = [
    ("tiny", dict(T=200)),                              # fp32 CUDA-core route, d = 32
    ("gdn", dict(B=1, H=2, T=300)),                     # Gated-DeltaNet tensor-core route
    ("long", dict(H=2, T=300)),                         # fused rank-L route, d = 128, chunk 128
    ("recsys", dict(B=1, H=2, T=200)),                  # fused rank-L route, d = 64, L = 4
]


@pytest.mark.parametrize("name,over", ELEMENT_CASES)
def test_segment_element_matches_oracle(name, over):
    from delta_rule_sequence_b200.prism import prism_scan_segment_element

    wl = WORKLOADS[name].with_(**over)
    x = make_inputs(wl, seed=23)
    d = to_device(x)
    E, f = prism_scan_segment_element(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["u"], d["w"],
                                      chunk=wl.chunk)
    torch.cuda.synchronize()
    E_ref, f_ref = _oracle_element(x)
    compare("E", E.cpu().numpy(), E_ref, TOL[wl.io])
    compare("f", f.cpu().numpy(), f_ref, TOL[wl.io])


def test_segment_element_of_no_tokens_is_the_identity():
    from delta_rule_sequence_b200.prism import prism_scan_segment_element

    wl = WORKLOADS["gdn"].with_(B=1, H=2, T=0)
    d = to_device(make_inputs(wl, seed=1))
    E, f = prism_scan_segment_element(d["q"], d["k"], d["v"], d["alpha"], d["beta"], chunk=64)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(E.cpu().numpy(), np.broadcast_to(np.eye(128), E.shape))
    np.testing.assert_array_equal(f.cpu().numpy(), 0.0)


@pytest.mark.parametrize("dk,dv,BH", [(128, 128, 5), (64, 64, 3), (32, 32, 7), (128, 64, 2)])
def test_state_fold_matches_fp64(dk, dv, BH):
    from delta_rule_sequence_b200.prism import prism_state_fold

    g = torch.Generator().manual_seed(dk + dv + BH)
    S = torch.randn((BH, dv, dk), generator=g)
    E = torch.randn((BH, dk, dk), generator=g) / dk ** 0.5
    f = torch.randn((BH, dv, dk), generator=g)
    ref = S.double().numpy() @ E.double().numpy() + f.double().numpy()
    out = prism_state_fold(S.cuda(), E.cuda(), f.cuda())
    torch.cuda.synchronize()
    compare("S E + f", out.cpu().numpy(), ref, TOL["f32"])
    # no entry state: the fold is f itself; in place: S_out may be S_in
    z = prism_state_fold(None, E.cuda(), f.cuda())
    Sd = S.cuda()
    prism_state_fold(Sd, E.cuda(), f.cuda(), S_out=Sd)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(z.cpu().numpy(), f.numpy())
    compare("in place", Sd.cpu().numpy(), ref, TOL["f32"])


@pytest.mark.parametrize("name,over,cut", [
    ("gdn", dict(B=1, H=2, T=512, s0_std=0.02), 256),
    ("gdn", dict(B=1, H=2, T=333), 140),                # cut inside a chunk, ragged end
    ("long", dict(H=2, T=512), 256),                     # rank-L, nonzero S0
])
def test_two_segments_the_way_two_ranks_run_them(name, over, cut):
    from delta_rule_sequence_b200 import prism

    wl = WORKLOADS[name].with_(**over)
    x = make_inputs(wl, seed=29)
    d = to_device(x)
    seg = [{n: (None if t is None or n == "S0" else t[:, a:b].contiguous()) for n, t in d.items()}
           for a, b in ((0, cut), (cut, wl.T))]
    p0, p1 = seg
    E0, f0 = prism.prism_scan_segment_element(p0["q"], p0["k"], p0["v"], p0["alpha"], p0["beta"],
                                              p0["u"], p0["w"], chunk=wl.chunk)
    entry = prism.prism_state_fold(d["S0"], E0, f0)
    o0, S0_exit = prism.prism_scan_fwd(p0["q"], p0["k"], p0["v"], p0["alpha"], p0["beta"], p0["u"],
                                       p0["w"], d["S0"], chunk=wl.chunk)
    o1, S_fin = prism.prism_scan_fwd(p1["q"], p1["k"], p1["v"], p1["alpha"], p1["beta"], p1["u"],
                                     p1["w"], entry, chunk=wl.chunk)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.scan_ref(**x)
    tol = TOL[wl.io]
    compare("entry state (fold of segment 0)", entry.cpu().numpy(), S0_exit.cpu().numpy(), tol)
    compare("o", torch.cat([o0, o1], 1).float().cpu().numpy(), o_ref, tol)
    compare("S_final", S_fin.cpu().numpy(), S_ref, tol)
