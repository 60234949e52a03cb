"""GPU parity on the method's edge regimes: the CUDA path (through the C ABI) against the fp64
oracle, element by element, at the standard tolerances (bf16 I/O 2e-2, fp32 I/O 1e-4, an element
passes iff |x - r| <= tol (1 + |r|)).

The regimes are the special cases the pages' recurrence reduces to, plus its numerical extremes
(banbantang.com PRISM article, section 1(4): scalar decay, rank-1 erase along k, rank-1 write;
"Sequential Parallel Duality in Prefix Scannable Models" (papernotes), key design 2: any chunking
of the affine elements gives the same result):

  - alpha = 1, beta = 0: causal linear attention (no decay, no erase; the state only grows);
  - beta = 0: gated linear attention with the rank-L write;
  - alpha = beta = 1 with q = k and exactly-unit keys: the full overwrite, o_t = v_t;
  - strong decay, alpha in [0.01, 0.2]: e^{g} underflows to zero inside a chunk;
  - beta = 1 everywhere: every step erases its key direction completely;
  - a large entry state (std 1);
  - write directions of norm ~8 and keys slightly off unit norm (the state grows into the tens
    or hundreds, where the state kernel switches its Wk_lo precision term on).

Every case runs on the Gated-DeltaNet route (u, w absent) and on the rank-L route, at bf16 on the
tensor-core kernels (d = 64 and 128) and at fp32 on the CUDA-core kernel, over T = 200 tokens
(three 64-token chunks and a ragged tail).  At d = 128 the state kernel splits the value columns
into slices of 16 when there are few sequences and of 32 otherwise (the slice width follows from
B H and the SM count); the d = 128 bf16 cases run once with two heads (16-wide slices) and once
with enough heads for 32-wide ones."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from delta_rule_sequence_b200.workloads import WORKLOADS, make_inputs
from tests.parity import check_scan_full

pytestmark = pytest.mark.gpu

FORCE_WK_LO = 16  # prism_debug_set_flags bit 4


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from delta_rule_sequence_b200 import build

    build.build()


# (route, d, L, io): the Gated-DeltaNet write (L = 1, u = w = None) or the projected rank-L write
ROUTES = [("gdn", 128, 1, "bf16"), ("gdn", 64, 1, "bf16"), ("gdn", 32, 1, "f32"),
          ("rank", 128, 2, "bf16"), ("rank", 64, 3, "bf16"), ("rank", 64, 2, "f32")]
T = 200


def _heads_for_wide_slices():
    """Enough heads that 16-wide value slices at d = 128 would outnumber the SMs."""
    return torch.cuda.get_device_properties(0).multi_processor_count // 8 + 1


def _base(route, d, L, io, seed, H=2):
    wl = WORKLOADS["gdn" if route == "gdn" else "recsys"].with_(
        B=1, H=H, T=T, dk=d, dv=d, L=L, io=io, s0_std=0.0)
    return wl, make_inputs(wl, seed=seed)


def _exact_unit_keys(g, B, T, H, d):
    """Keys with four entries of +-1/2 and the rest zero: norm exactly 1 in any binary format."""
    k = torch.zeros((B, T, H, d))
    for idx in np.ndindex(B, T, H):
        pos = torch.randperm(d, generator=g)[:4]
        sgn = torch.randint(0, 2, (4,), generator=g).float() * 2 - 1
        k[idx][pos] = 0.5 * sgn
    return k


def _edge(x, wl, case, seed):
    """Modify a seeded batch into one of the edge regimes (in place on CPU tensors)."""
    g = torch.Generator().manual_seed(1000 + seed)
    io = wl.torch_io
    B, T_, H, d = x["q"].shape
    if case == "linear_attention":
        x["alpha"][:] = 1.0
        x["beta"][:] = 0.0
        if x["u"] is not None:  # rank-L route: its L = 1 form u = v, w = k is the closed form
            v = torch.randn((B, T_, H, d), generator=g).to(io)
            x["u"] = v[:, :, :, None, :].repeat(1, 1, 1, wl.L, 1).contiguous()
            x["w"] = x["k"][:, :, :, None, :].repeat(1, 1, 1, wl.L, 1).contiguous()
    elif case == "gla":
        x["beta"][:] = 0.0
    elif case == "overwrite":
        k = _exact_unit_keys(g, B, T_, H, d).to(io)
        x["k"] = k
        x["q"] = k.clone()
        x["alpha"][:] = 1.0
        x["beta"][:] = 1.0
        if x["u"] is not None:  # the overwrite through the rank-L route: u = v (beta = 1), w = k
            v = torch.randn((B, T_, H, d), generator=g).to(io)
            u = torch.zeros((B, T_, H, wl.L, d), dtype=io)
            w = torch.zeros((B, T_, H, wl.L, d), dtype=io)
            u[:, :, :, 0] = v
            w[:, :, :, 0] = k
            x["u"], x["w"] = u, w
    elif case == "strong_decay":
        x["alpha"] = (0.01 + 0.19 * torch.rand((B, T_, H), generator=g)).float()
    elif case == "beta_one":
        x["beta"][:] = 1.0
    elif case == "big_state":
        x["S0"] = torch.randn((B, H, d, d), generator=g).float()
    elif case == "large_directions":
        # write directions of norm ~8 (as an unnormalised W_k^(l) anchor projection gives) and
        # keys 5 % off unit norm
        scale = 1.0 + 0.05 * torch.randn((B, T_, H, 1), generator=g)
        x["k"] = (x["k"].float() * scale).to(io)
        if x["u"] is not None:
            w = x["w"].float()
            x["w"] = (8.0 * w / w.norm(dim=-1, keepdim=True)).to(io)
            x["u"] = (x["u"].float() * 4.0).to(io)
        else:
            x["v"] = (x["v"].float() * 8.0).to(io)
    else:
        raise ValueError(case)
    return x


CASES = ["linear_attention", "gla", "overwrite", "strong_decay", "beta_one", "big_state",
         "large_directions"]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("route,d,L,io", ROUTES)
def test_edge_regime_matches_oracle(case, route, d, L, io):
    seed = CASES.index(case) * 7 + d + L
    wl, x = _base(route, d, L, io, seed)
    x = _edge(x, wl, case, seed)
    check_scan_full(x, wl.chunk, io)


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("route,L", [("gdn", 1), ("rank", 2)])
def test_edge_regime_32_wide_slices(case, route, L):
    """The same regimes at d = 128 with enough heads for the 32-wide value slices."""
    seed = CASES.index(case) * 7 + 128 + L + 1
    wl, x = _base(route, 128, L, "bf16", seed, H=_heads_for_wide_slices())
    x = _edge(x, wl, case, seed)
    check_scan_full(x, wl.chunk, "bf16")


def test_overwrite_returns_the_values():
    """alpha = beta = 1, q = k with exactly-unit keys: o_t = v_t (read back what was just written)."""
    from delta_rule_sequence_b200.prism import prism_scan_fwd

    wl, x = _base("gdn", 128, 1, "bf16", 5)
    x = _edge(x, wl, "overwrite", 5)
    d = {n: (None if t is None else t.cuda()) for n, t in x.items()}
    o, _ = prism_scan_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], chunk=64)
    torch.cuda.synchronize()
    ref = x["v"].float()
    err = (o.float().cpu() - ref).abs() - 2e-2 * (1 + ref.abs())
    assert (err <= 0).all(), float(err.max())


def test_state_growth_beyond_one_hundred_matches_oracle():
    """No decay, no erase and write directions of norm 8: the state grows as sqrt(T) into the
    tens and hundreds; the Wk_lo term must keep every output element within tolerance."""
    wl = WORKLOADS["recsys"].with_(B=1, H=2, T=600, dk=64, dv=64, L=3, s0_std=0.0)
    x = make_inputs(wl, seed=21)
    x["alpha"][:] = 1.0
    x["beta"][:] = 0.0
    w = x["w"].float()
    x["w"] = (8.0 * w / w.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    x["u"] = (x["u"].float() * 4.0).to(torch.bfloat16)
    import oracle

    _, S_ref = oracle.scan_ref(**x)
    assert np.abs(S_ref).max() > 50.0  # the regime is really reached
    check_scan_full(x, wl.chunk, wl.io)
    wl2 = WORKLOADS["long"].with_(H=2, T=450, L=2, chunk=64, s0_std=0.0)
    x2 = make_inputs(wl2, seed=22)
    x2["alpha"][:] = 1.0
    x2["beta"][:] = 0.0
    w2 = x2["w"].float()
    x2["w"] = (8.0 * w2 / w2.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    x2["u"] = (x2["u"].float() * 4.0).to(torch.bfloat16)
    check_scan_full(x2, wl2.chunk, wl2.io)


@pytest.mark.parametrize("name,over", [
    ("gdn", dict(B=2, H=2, T=300)),
    ("gdn", dict(B=1, H=3, T=200, dk=64, dv=64)),
    ("recsys", dict(B=2, H=2, T=200)),
    ("long", dict(H=2, T=333, chunk=64)),
])
def test_forced_wk_lo_term_matches_oracle(name, over):
    """The Wk_lo term switched on from the first chunk (debug flag): X_s gains it and the Q S rows
    of the same accumulator are left untouched by the lane-masked MMAs."""
    from delta_rule_sequence_b200 import prism

    lib = prism.load_library()
    wl = WORKLOADS[name].with_(**over)
    x = make_inputs(wl, seed=31)
    old = lib.prism_debug_set_flags(FORCE_WK_LO)
    try:
        check_scan_full(x, wl.chunk, wl.io)
    finally:
        lib.prism_debug_set_flags(old)
