"""Failure detection without a GPU fault.  A debug flag makes one kernel's load role issue nothing,
so every bounded wait in that kernel runs out after a short limit; the kernel must record
PRISM_ERR_TIMEOUT in its status word (the workspace's for the scan kernels, the library's own for
the producer and the decode step), return without hanging, and leave the context usable: reading
the status clears it, and the next call on the same context is correct.

Stall flags (prism_debug_set_flags): 8 the in-order state kernel, 32 the per-chunk prep kernels,
64 the write producer, 128 the bulk-copy decode kernel."""
import ctypes

import pytest
import torch

import oracle
from oracle.write_producer import write_producer_ref
from delta_rule_sequence_b200.workloads import (WORKLOADS, make_decode_state, make_decode_step,
                                                 make_inputs, make_producer_inputs)
from tests.parity import TOL, check_scan_full, compare, to_device

pytestmark = pytest.mark.gpu

STALL_STATE, STALL_PREP, STALL_PRODUCER, STALL_DECODE = 8, 32, 64, 128
FORCE_SEGMENTS = 2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from delta_rule_sequence_b200 import build

    build.build()


def _with_flags(flags, fn):
    from delta_rule_sequence_b200 import prism

    lib = prism.load_library()
    old = lib.prism_debug_set_flags(flags)
    try:
        return fn()
    finally:
        lib.prism_debug_set_flags(old)


def _stalled_scan(wl, flags, seed=3):
    """One scan with `flags` set; returns the status read from its workspace twice."""
    from delta_rule_sequence_b200 import prism

    lib = prism.load_library()
    d = to_device(make_inputs(wl, seed=seed))

    def run():
        shape = prism.make_shape(d["q"], d["v"], d["u"], wl.chunk)
        need = ctypes.c_size_t(0)
        assert lib.prism_scan_fwd_workspace_size(ctypes.byref(shape), ctypes.byref(need)) == 0
        ws = torch.zeros(int(need.value), dtype=torch.uint8, device="cuda")
        prism.prism_scan_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["u"], d["w"],
                             d["S0"], chunk=wl.chunk, workspace=ws)
        return prism.prism_query_device_status(ws), prism.prism_query_device_status(ws)

    return _with_flags(flags, run)


@pytest.mark.parametrize("name,flags", [
    ("gdn", STALL_STATE),     # Gated-DeltaNet state kernel
    ("gdn", STALL_PREP),      # gdn_prep_kernel
    ("long", STALL_STATE),    # rank-L state kernel
    ("long", STALL_PREP),     # lrank_prep_kernel
    ("long", STALL_STATE | FORCE_SEGMENTS),  # the segmented scan's passes
    ("gdn", STALL_PREP | FORCE_SEGMENTS),
])
def test_scan_kernels_give_up_and_report_a_timeout(name, flags):
    from delta_rule_sequence_b200 import prism

    wl = WORKLOADS[name].with_(B=1, H=2, T=256, chunk=64)
    first, second = _stalled_scan(wl, flags)
    assert first == prism.PRISM_ERR_TIMEOUT
    assert second == prism.PRISM_OK  # read and cleared
    # the context is still usable: the same shape now runs correctly
    check_scan_full(make_inputs(wl, seed=4), wl.chunk, wl.io)


@pytest.mark.parametrize("d", [64, 128])
def test_producer_gives_up_and_reports_a_timeout(d):
    from delta_rule_sequence_b200 import prism

    wl = WORKLOADS["recsys"].with_(B=1, H=2, T=200, L=3, dk=d, dv=d)
    p = to_device(make_producer_inputs(wl, seed=5))
    call = lambda: prism.prism_write_producer(p["x"], p["v"], p["conv"], p["Wk"], p["Wp"], p["beta"])
    _with_flags(STALL_PRODUCER, call)
    assert prism.prism_query_device_status(None) == prism.PRISM_ERR_TIMEOUT
    assert prism.prism_query_device_status(None) == prism.PRISM_OK
    u, w = call()
    torch.cuda.synchronize()
    u_ref, w_ref, _ = write_producer_ref(**make_producer_inputs(wl, seed=5))
    compare("u", u.float().cpu().numpy(), u_ref, TOL["bf16"])
    compare("w", w.float().cpu().numpy(), w_ref, TOL["bf16"])


def test_decode_gives_up_and_reports_a_timeout():
    from delta_rule_sequence_b200 import prism

    wl = WORKLOADS["decode"].with_(B=4, H=2)
    st = make_decode_state(wl)
    x = make_decode_step(wl, st, 0)
    d = to_device(x)
    S = st["S0"].cuda()
    step = lambda: prism.prism_step_decode(d["q"], d["k"], None, d["alpha"], d["beta"], d["u"],
                                           d["w"], S)
    _with_flags(STALL_DECODE, step)
    assert prism.prism_query_device_status(None) == prism.PRISM_ERR_TIMEOUT
    assert prism.prism_query_device_status(None) == prism.PRISM_OK
    assert torch.equal(S.cpu(), st["S0"])  # a step that gave up leaves the state untouched
    o = step()
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.scan_ref(**x, S0=st["S0"])
    compare("o", o.float().cpu().numpy(), o_ref, TOL["bf16"])
    compare("S", S.cpu().numpy(), S_ref, TOL["bf16"])
