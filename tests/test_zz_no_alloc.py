"""prism_scan_fwd_noalloc: the scan for callers that cannot allocate device memory when they run it
(engine plugins that own every allocation, latency-critical paths that cannot take cudaMalloc's
synchronisation).  It runs on the library's own fixed device scratch instead of a caller
workspace.  Checked here through the C ABI, for two calls in a row (the second call reuses the
scratch the first one left behind), against prism_scan_fwd on the same inputs and against the
fp64 oracle; its argument checks against prism_scan_fwd's; and its status word (in the scratch)
through prism_query_device_status.

This file is collected last on purpose, so that a run which stops at the first failure has
already run every other test."""
import ctypes

import pytest
import torch

import oracle
from delta_rule_sequence_b200.workloads import WORKLOADS, make_inputs
from tests.parity import TOL, compare, to_device

pytestmark = pytest.mark.gpu

STALL_TEST = 8  # prism_debug_set_flags bit 3


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
        x = make_inputs(wl, seed=seed)
        o, S, o_ws, S_ws = _both(x, wl.chunk)
        compare(f"o vs prism_scan_fwd (call {call})", o.float().cpu().numpy(),
                o_ws.float().cpu().numpy(), tol)
        compare(f"S_final vs prism_scan_fwd (call {call})", S.cpu().numpy(), S_ws.cpu().numpy(), tol)
        o_ref, S_ref = oracle.scan_ref(**x)
        compare(f"o vs oracle (call {call})", o.float().cpu().numpy(), o_ref, tol)
        compare(f"S_final vs oracle (call {call})", S.cpu().numpy(), S_ref, tol)


def test_noalloc_rejects_bad_arguments_like_the_workspace_entry():
    """Real (small) device buffers everywhere, so that a check that stopped rejecting would give a
    wrong status here, never a launch on a bad address."""
    from delta_rule_sequence_b200 import prism as P

    lib = P.load_library()
    buf = torch.zeros(1 << 16, dtype=torch.float32, device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    p = ctypes.c_void_p(buf.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    bad = [
        (P.PrismShape(1, 2, 64, 48, 48, 1, 64, P.PRISM_BF16), P.PRISM_ERR_UNSUPPORTED),  # width
        (P.PrismShape(-1, 2, 64, 64, 64, 1, 64, P.PRISM_BF16), P.PRISM_ERR_INVALID_ARG),  # B < 0
        (P.PrismShape(1, 2, 64, 64, 64, 1, 32, P.PRISM_BF16), P.PRISM_ERR_INVALID_ARG),   # chunk
        (P.PrismShape(1, 2, 64, 64, 64, 0, 64, P.PRISM_BF16), P.PRISM_ERR_INVALID_ARG),   # L < 1
        (P.PrismShape(1, 2, 64, 64, 64, 9, 64, P.PRISM_BF16), P.PRISM_ERR_UNSUPPORTED),   # L > 8
    ]
    for shape, code in bad:
        rc_na = lib.prism_scan_fwd_noalloc(ctypes.byref(shape), p, p, p, p, p, None, None, None, p,
                                           None, stream)
        rc_ws = lib.prism_scan_fwd(ctypes.byref(shape), p, p, p, p, p, None, None, None, p, None,
                                   ctypes.c_void_p(ws.data_ptr()), ctypes.c_size_t(ws.numel()), stream)
        assert rc_na == rc_ws == code, (shape.B, shape.dk, shape.chunk, shape.L, rc_na, rc_ws)
    assert lib.prism_scan_fwd_noalloc(None, *([None] * 10), None) == P.PRISM_ERR_INVALID_ARG
    torch.cuda.synchronize()


def test_noalloc_status_word_is_reported_and_cleared():
    """A bounded wait that gives up inside a no-alloc call is recorded in the scratch's status word;
    prism_query_device_status(NULL) reports and clears it, and the next call is correct."""
    from delta_rule_sequence_b200 import prism as P

    lib = P.load_library()
    wl = WORKLOADS["gdn"].with_(B=1, H=2, T=256)
    d = to_device(make_inputs(wl, seed=3))
    o = torch.empty((1, 256, 2, 128), dtype=torch.bfloat16, device="cuda")
    S = torch.empty((1, 2, 128, 128), dtype=torch.float32, device="cuda")
    assert P.prism_query_device_status(None) == P.PRISM_OK
    old = lib.prism_debug_set_flags(STALL_TEST)
    try:
        P.prism_scan_fwd_noalloc(d["q"], d["k"], d["v"], d["alpha"], d["beta"], chunk=64, o=o,
                                 S_final=S)
        assert P.prism_query_device_status(None) == P.PRISM_ERR_TIMEOUT
        assert P.prism_query_device_status(None) == P.PRISM_OK  # read and cleared
    finally:
        lib.prism_debug_set_flags(old)
    o2, S2, _, _ = _both(make_inputs(wl, seed=4), 64)
    o_ref, S_ref = oracle.scan_ref(**make_inputs(wl, seed=4))
    compare("o after the stall", o2.float().cpu().numpy(), o_ref, TOL["bf16"])
    compare("S_final after the stall", S2.cpu().numpy(), S_ref, TOL["bf16"])
