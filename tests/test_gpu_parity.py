"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same seeded inputs.

Reduced sizes compare every element and span several chunks plus a ragged tail; full sizes run
the launch configuration the bench times and compare sampled (b, h) sequences.  Tolerances:
2e-2 for bf16 I/O, 1e-4 for fp32 I/O, element-wise |x - r| <= tol (1 + |r|)."""
import pytest
import torch

import oracle
from delta_rule_sequence_b200.workloads import (WORKLOADS, make_decode_state, make_decode_step,
                                                 make_inputs, select_heads)
from tests.parity import TOL, check_scan_full, check_scan_sampled, compare, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from delta_rule_sequence_b200 import build

    build.build()


# ---------------------------------------------------------------------------------------------
# reduced sizes: every element

def test_tiny_config_fp32_full():
    wl = WORKLOADS["tiny"]
    check_scan_full(make_inputs(wl), wl.chunk, wl.io)


@pytest.mark.parametrize("T", [1, 63, 64, 300])
def test_gdn_reduced(T):
    wl = WORKLOADS["gdn"].with_(B=2, H=2, T=T)
    check_scan_full(make_inputs(wl, seed=T), wl.chunk, wl.io)


@pytest.mark.parametrize("T", [5, 200])
def test_recsys_reduced(T):
    wl = WORKLOADS["recsys"].with_(B=2, H=2, T=T)
    check_scan_full(make_inputs(wl, seed=T), wl.chunk, wl.io)


def test_long_reduced_nonzero_state():
    wl = WORKLOADS["long"].with_(H=2, T=333)
    check_scan_full(make_inputs(wl), wl.chunk, wl.io)


@pytest.mark.parametrize("dk,L,io", [(32, 1, "bf16"), (64, 3, "f32"), (128, 4, "f32"),
                                      (32, 8, "bf16")])
def test_other_widths_and_ranks(dk, L, io):
    wl = WORKLOADS["recsys"].with_(B=1, H=3, T=150, dk=dk, dv=dk, L=L, io=io)
    check_scan_full(make_inputs(wl, seed=dk + L), wl.chunk, io)


@pytest.mark.parametrize("dk,T", [(64, 200), (128, 77)])
def test_gdn_write_bf16_widths(dk, T):
    wl = WORKLOADS["gdn"].with_(B=2, H=3, T=T, dk=dk, dv=dk)
    check_scan_full(make_inputs(wl, seed=dk), wl.chunk, wl.io)


@pytest.mark.parametrize("dk,L,T", [(128, 8, 130), (64, 1, 64), (128, 3, 1), (64, 3, 200),
                                    (64, 5, 129), (128, 2, 257)])
def test_rank_l_write_bf16(dk, L, T):
    wl = WORKLOADS["long"].with_(H=2, T=T, dk=dk, dv=dk, L=L, chunk=64)
    check_scan_full(make_inputs(wl, seed=L), wl.chunk, wl.io)


def test_empty_sequence_copies_state():
    wl = WORKLOADS["long"].with_(H=2, T=1)
    x = make_inputs(wl)
    from delta_rule_sequence_b200.prism import prism_scan_fwd

    d = to_device(x)
    q0 = d["q"][:, :0].contiguous()
    k0 = d["k"][:, :0].contiguous()
    u0 = d["u"][:, :0].contiguous()
    w0 = d["w"][:, :0].contiguous()
    a0 = d["alpha"][:, :0].contiguous()
    b0 = d["beta"][:, :0].contiguous()
    o, Sf = prism_scan_fwd(q0, k0, None, a0, b0, u0, w0, d["S0"], chunk=128)
    torch.cuda.synchronize()
    assert o.shape[1] == 0
    assert torch.equal(Sf.cpu(), x["S0"])


def test_gdn_route_matches_general_route_on_gpu():
    wl = WORKLOADS["gdn"].with_(B=1, H=2, T=130)
    x = make_inputs(wl)
    d = to_device(x)
    from delta_rule_sequence_b200.prism import prism_scan_fwd

    o1, S1 = prism_scan_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], chunk=64)
    u = (d["beta"][..., None].float() * d["v"].float()).to(d["v"].dtype)[:, :, :, None, :]
    w = d["k"][:, :, :, None, :].contiguous()
    o2, S2 = prism_scan_fwd(d["q"], d["k"], None, d["alpha"], d["beta"], u.contiguous(), w,
                            chunk=64)
    torch.cuda.synchronize()
    # u = beta v is rounded to bf16 on the general route, so compare at the bf16 tolerance
    compare("o", o2.float().cpu().numpy(), o1.float().cpu().numpy(), TOL["bf16"])
    compare("S", S2.cpu().numpy(), S1.cpu().numpy(), TOL["bf16"])


def test_resume_from_state_matches_one_pass():
    wl = WORKLOADS["long"].with_(H=2, T=300)
    x = make_inputs(wl)
    d = to_device(x)
    from delta_rule_sequence_b200.prism import prism_scan_fwd

    o, S = prism_scan_fwd(d["q"], d["k"], None, d["alpha"], d["beta"], d["u"], d["w"], d["S0"],
                          chunk=128)
    for T1 in (128, 77):
        sl = lambda n, a, b: d[n][:, a:b].contiguous()
        o1, S1 = prism_scan_fwd(sl("q", 0, T1), sl("k", 0, T1), None, sl("alpha", 0, T1),
                                sl("beta", 0, T1), sl("u", 0, T1), sl("w", 0, T1), d["S0"],
                                chunk=128)
        o2, S2 = prism_scan_fwd(sl("q", T1, 300), sl("k", T1, 300), None, sl("alpha", T1, 300),
                                sl("beta", T1, 300), sl("u", T1, 300), sl("w", T1, 300), S1,
                                chunk=128)
        torch.cuda.synchronize()
        compare("o", torch.cat([o1, o2], 1).float().cpu().numpy(), o.float().cpu().numpy(),
                TOL["bf16"])
        compare("S", S2.cpu().numpy(), S.cpu().numpy(), TOL["bf16"])


def test_launch_probe_brackets_every_launch():
    """The events that prism_debug_record_launch_events arms are recorded around each launch of
    the next call only (the bench times its kernels with them)."""
    from delta_rule_sequence_b200 import prism

    wl = WORKLOADS["gdn"].with_(B=1, H=2, T=512)
    d = to_device(make_inputs(wl))
    shape = prism.make_shape(d["q"], d["v"], None, wl.chunk)
    n = prism.prism_scan_fwd_launch_count(shape)
    assert n == 2
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
    for e in evs:
        e.record()
    torch.cuda.synchronize()
    marker = torch.cuda.Event(enable_timing=True)
    marker.record()
    prism.record_launch_events(evs)
    prism.prism_scan_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], chunk=wl.chunk)
    prism.prism_scan_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], chunk=wl.chunk)
    torch.cuda.synchronize()
    assert marker.elapsed_time(evs[0]) >= 0.0  # recorded after the marker, i.e. re-recorded
    for j in range(n):
        assert evs[j].elapsed_time(evs[j + 1]) > 0.0


# ---------------------------------------------------------------------------------------------
# full sizes, in the launch configuration the bench uses; sampled sequences

def test_gdn_full_size_sampled():
    wl = WORKLOADS["gdn"]
    check_scan_sampled(make_inputs(wl), wl.chunk, wl.io, [(0, 0), (1, 5), (2, 3), (3, 7)])


def test_recsys_full_size_sampled():
    wl = WORKLOADS["recsys"]
    check_scan_sampled(make_inputs(wl), wl.chunk, wl.io, [(0, 0), (13, 2), (31, 3)])


def test_long_full_size_sampled():
    wl = WORKLOADS["long"]
    check_scan_sampled(make_inputs(wl), wl.chunk, wl.io, [(0, 0), (0, 9), (0, 15)])


# ---------------------------------------------------------------------------------------------
# decode step

def _decode_run(wl, steps, heads_to_keep=None):
    """Run `steps` consecutive decode steps on the GPU; return per-step outputs of the kept
    heads, their inputs (stacked along T, as the oracle takes them) and the final state."""
    from delta_rule_sequence_b200.prism import prism_step_decode

    st = make_decode_state(wl)
    S = st["S0"].cuda()
    kept_o, kept_in = [], []
    for s in range(steps):
        x = make_decode_step(wl, st, s)
        d = to_device(x)
        o = prism_step_decode(d["q"], d["k"], None, d["alpha"], d["beta"], d["u"], d["w"], S)
        if heads_to_keep is None:
            kept_o.append(o.float().cpu())
            kept_in.append(x)
        else:
            kept_o.append(torch.cat([o[b:b + 1, :, h:h + 1] for b, h in heads_to_keep], 0)
                          .float().cpu())
            kept_in.append(select_heads(x, heads_to_keep))
    torch.cuda.synchronize()
    stacked = {n: (None if kept_in[0][n] is None else torch.cat([y[n] for y in kept_in], 1))
               for n in kept_in[0] if n != "S0"}
    return torch.cat(kept_o, 1).numpy(), stacked, S.cpu(), st["S0"]


def test_decode_full_size_all_heads_10_steps():
    wl = WORKLOADS["decode"]
    o, xin, S, S0 = _decode_run(wl, 10)
    o_ref, S_ref = oracle.scan_ref(**xin, S0=S0)
    compare("o", o, o_ref, TOL["bf16"])
    compare("S", S.numpy(), S_ref, TOL["bf16"])


def test_decode_1000_steps_sampled_heads():
    wl = WORKLOADS["decode"]
    heads = [(0, 0), (77, 31), (255, 12)]
    o, xin, S, S0 = _decode_run(wl, 1000, heads)
    S0s = torch.cat([S0[b:b + 1, h:h + 1] for b, h in heads], 0)
    o_ref, S_ref = oracle.scan_ref(**xin, S0=S0s)
    compare("o", o, o_ref, TOL["bf16"])
    S_got = torch.cat([S[b:b + 1, h:h + 1] for b, h in heads], 0).numpy()
    compare("S", S_got, S_ref, TOL["bf16"])


@pytest.mark.parametrize("dk,L,io,gdn", [(32, 1, "f32", True), (64, 3, "bf16", False),
                                          (128, 8, "f32", False)])
def test_decode_other_shapes(dk, L, io, gdn):
    from delta_rule_sequence_b200.prism import prism_step_decode

    wl = WORKLOADS["recsys"].with_(B=3, H=2, T=1, dk=dk, dv=dk, L=L, io=io,
                                   write="gdn" if gdn else "projected", s0_std=0.05)
    x = make_inputs(wl)
    d = to_device(x)
    S = d["S0"].clone()
    o = prism_step_decode(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["u"], d["w"], S)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.scan_ref(**x)
    compare("o", o.float().cpu().numpy(), o_ref, TOL[io])
    compare("S", S.cpu().numpy(), S_ref, TOL[io])
