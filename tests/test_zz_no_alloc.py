"""prism_scan_fwd_noalloc: the scan for callers that cannot allocate device memory when they run it
(engine plugins that own every allocation, latency-critical paths that cannot take cudaMalloc's
synchronisation).  It runs on the library's own fixed device scratch instead of a caller
workspace.  Checked here through the C ABI against prism_scan_fwd on the same inputs, for two
calls in a row (the second call reuses the scratch the first one left behind).

This file is collected last on purpose, so that a run which stops at the first failure has
already run every other test."""
import pytest
import torch

from delta_rule_sequence_b200.workloads import WORKLOADS, make_inputs
from tests.parity import TOL, compare, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from delta_rule_sequence_b200 import build

    build.build()


def _both(x, chunk):
    from delta_rule_sequence_b200.prism import prism_scan_fwd, prism_scan_fwd_noalloc

    d = to_device(x)
    o_ref, S_ref = prism_scan_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["u"], d["w"],
                                  d["S0"], chunk=chunk)
    o = torch.empty_like(o_ref)
    S = torch.empty_like(S_ref)
    prism_scan_fwd_noalloc(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["u"], d["w"],
                           d["S0"], chunk=chunk, o=o, S_final=S)
    torch.cuda.synchronize()
    return o, S, o_ref, S_ref


@pytest.mark.parametrize("name,over", [
    ("gdn", dict(B=2, H=2, T=300)),
    ("long", dict(H=2, T=200, chunk=64)),
])
def test_noalloc_matches_workspace_entry_two_calls(name, over):
    wl = WORKLOADS[name].with_(**over)
    tol = TOL[wl.io]
    for call, seed in enumerate((11, 12)):  # two calls in a row on the shared scratch
        o, S, o_ref, S_ref = _both(make_inputs(wl, seed=seed), wl.chunk)
        compare(f"o (call {call})", o.float().cpu().numpy(), o_ref.float().cpu().numpy(), tol)
        compare(f"S_final (call {call})", S.cpu().numpy(), S_ref.cpu().numpy(), tol)


def test_noalloc_rejects_bad_arguments_before_launch():
    import ctypes

    from delta_rule_sequence_b200 import prism as P

    lib = P.load_library()
    shape = P.PrismShape(1, 2, 64, 48, 48, 1, 64, P.PRISM_BF16)  # dk = 48 is not built
    fake = ctypes.c_void_p(0x10000)
    rc = lib.prism_scan_fwd_noalloc(ctypes.byref(shape), fake, fake, fake, fake, fake, None,
                                    None, None, fake, None, None)
    assert rc == P.PRISM_ERR_UNSUPPORTED
    assert lib.prism_scan_fwd_noalloc(None, *([None] * 10), None) == P.PRISM_ERR_INVALID_ARG
