"""GPU parity of the segmented inter-chunk scan (segment elements, a Blelloch scan over them, a
re-run of every segment from its entry state), forced on through prism_debug_set_flags so that it
is exercised on shapes small enough for the oracle.  Each case is checked element by element
against the fp64 oracle and against the one-pass result."""
import pytest
import torch

import oracle
from delta_rule_sequence_b200.workloads import WORKLOADS, make_inputs
from tests.parity import TOL, compare, to_device

pytestmark = pytest.mark.gpu

FORCE, NEVER = 2, 4


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from delta_rule_sequence_b200 import build

    build.build()


@pytest.fixture
def flags():
    from delta_rule_sequence_b200 import prism

    lib = prism.load_library()
    old = lib.prism_debug_set_flags(0)
    yield lambda f: lib.prism_debug_set_flags(f)
    lib.prism_debug_set_flags(old)


def _run(x, chunk):
    from delta_rule_sequence_b200.prism import prism_scan_fwd

    d = to_device(x)
    o, S = prism_scan_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["u"], d["w"], d["S0"],
                          chunk=chunk, workspace=None)
    torch.cuda.synchronize()
    return o.float().cpu().numpy(), S.cpu().numpy()


CASES = [
    ("gdn", dict(B=1, H=2, T=1024, s0_std=0.02)),          # tensor-core GDN route, G = 16
    ("gdn", dict(B=2, H=1, T=640, s0_std=0.02)),           # segments of 80 tokens (ragged chunks)
    ("recsys", dict(B=2, H=1, T=512)),                     # fused rank-L route, d = 64, L = 4
    ("long", dict(H=2, T=2048)),                           # fused rank-L route, d = 128, L = 2
    ("tiny", dict(T=256, s0_std=0.05)),                    # fp32 CUDA-core route
]


@pytest.mark.parametrize("name,over", CASES)
def test_segmented_matches_oracle_and_one_pass(flags, name, over):
    from delta_rule_sequence_b200 import prism

    wl = WORKLOADS[name].with_(**over)
    x = make_inputs(wl, seed=17)
    tol = TOL[wl.io]
    flags(FORCE)
    shape = prism.make_shape(x["q"], x["v"], x["u"], wl.chunk)
    assert prism.prism_scan_fwd_launch_count(shape) > 2, "the segmented plan was not taken"
    prism._ws_cache.clear()
    o_seg, S_seg = _run(x, wl.chunk)
    flags(NEVER)
    prism._ws_cache.clear()
    o_one, S_one = _run(x, wl.chunk)
    o_ref, S_ref = oracle.scan_ref(**x)
    compare("o (segmented)", o_seg, o_ref, tol)
    compare("S_final (segmented)", S_seg, S_ref, tol)
    compare("o (segmented vs one pass)", o_seg, o_one, tol)
    compare("S_final (segmented vs one pass)", S_seg, S_one, tol)
