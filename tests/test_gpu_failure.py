"""Failure detection without a GPU fault: the stall test makes the Gated-DeltaNet state kernel's
load warp issue nothing, so every wait in the kernel runs out after a short limit; the kernel must
record PRISM_ERR_TIMEOUT in the workspace status word, return, and leave the context usable."""
import ctypes

import pytest
import torch

from delta_rule_sequence_b200.workloads import WORKLOADS, make_inputs
from tests.parity import check_scan_full, to_device

pytestmark = pytest.mark.gpu

STALL_TEST = 8


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from delta_rule_sequence_b200 import build

    build.build()


def test_state_kernel_gives_up_and_reports_a_timeout():
    from delta_rule_sequence_b200 import prism

    lib = prism.load_library()
    wl = WORKLOADS["gdn"].with_(B=1, H=2, T=256)
    d = to_device(make_inputs(wl, seed=3))
    shape = prism.make_shape(d["q"], d["v"], None, wl.chunk)
    need = ctypes.c_size_t(0)
    assert lib.prism_scan_fwd_workspace_size(ctypes.byref(shape), ctypes.byref(need)) == 0
    ws = torch.zeros(int(need.value), dtype=torch.uint8, device="cuda")
    old = lib.prism_debug_set_flags(STALL_TEST)
    try:
        prism.prism_scan_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], chunk=wl.chunk,
                             workspace=ws)
        assert prism.prism_query_device_status(ws) == prism.PRISM_ERR_TIMEOUT
        assert prism.prism_query_device_status(ws) == prism.PRISM_OK  # read and cleared
    finally:
        lib.prism_debug_set_flags(old)
    # the context is still usable: the same shape now runs correctly
    check_scan_full(make_inputs(wl, seed=4), wl.chunk, wl.io)
