"""GPU check of chunk-by-chunk streaming inference (delta_rule_sequence_b200.stream): the
library's segment element, fold and scan driven by the online binary counter, against one pass of
the fp64 oracle (bf16 tolerance |x - r| <= 2e-2 (1 + |r|))."""
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


@pytest.mark.parametrize("name,over,c", [
    ("gdn", dict(B=1, H=2, T=7 * 64, s0_std=0.02), 64),     # Gated-DeltaNet route, 7 chunks
    ("recsys", dict(B=1, H=2, T=5 * 64, L=3), 64),            # rank-L route, d = 64
])
def test_streaming_matches_oracle(name, over, c):
    from delta_rule_sequence_b200.stream import StreamingScan

    wl = WORKLOADS[name].with_(**over)
    x = make_inputs(wl, seed=17)
    d = to_device(x)
    s = StreamingScan(d["S0"], chunk=c)
    outs = []
    for t0 in range(0, wl.T, c):
        p = {n: (None if t is None or n == "S0" else t[:, t0:t0 + c].contiguous()) for n, t in d.items()}
        outs.append(s.step(p["q"], p["k"], p["v"], p["alpha"], p["beta"], p["u"], p["w"]))
    S = s.state()
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.scan_ref(**x)
    compare("o", torch.cat(outs, 1).float().cpu().numpy(), o_ref, TOL[wl.io])
    compare("S", S.cpu().numpy(), S_ref, TOL[wl.io])
    assert len(s.counter.live_roots()) == bin(wl.T // c).count("1")
