"""Seeded synthetic workloads for the scan forward and the decode step.

This module only draws inputs: it holds none of the method's arithmetic, and both the CUDA path
and the CPU oracle read the tensors it returns (the same bytes).  Every draw uses a CPU
``torch.Generator`` seeded explicitly, in a fixed tensor order, so that a workload is reproducible
on any host.

The shapes follow the workloads the pages describe: long user-behaviour sequences for sequential
recommendation (the PRISM pages' Amazon/Yelp benchmarks) and LM-style heads (SlimPajama language
modelling).  Those datasets are not available here; these synthetic tensors stand in for them.

Recipes (seed 0 for every workload):
  q, v ~ N(0, 1); k ~ N(0, 1) then L2-normalised per token.
  tiny:     alpha = exp(-0.1 softplus(N(0,1))),   beta = sigmoid(N(0,1)).
  others:   alpha = exp(-softplus(N(-3,1))),      beta = sigmoid(N(0,1)).
  projected writes (rank L): per (b,t,h) an anchor z ~ N(0, I_d); fixed per-(h,l) projections
            P_u, P_w with N(0, 1/d) entries; w_{t,l} = normalize(P_w z), u_{t,l} = 0.5^l P_u z.
  S0:       zero, or N(0, std^2) with std = 0.02 where the workload says so.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch
import torch.nn.functional as F


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    L: int
    chunk: int
    io: str            # "bf16" or "f32": type of q, k, v, u, w and of the output o
    write: str         # "gdn": u, w absent, the write is beta v k^T; "projected": rank-L u, w
    alpha_recipe: str  # "tiny" or "gdn"
    s0_std: float      # 0.0 means S0 is absent (zeros)
    steps: int = 0     # decode only: consecutive single-token steps

    @property
    def torch_io(self):
        return torch.float32 if self.io == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 256, 32, 32, 1, 64, "f32", "gdn", "tiny", 0.0),
    "gdn": Workload("gdn", 4, 8, 4096, 128, 128, 1, 64, "bf16", "gdn", "gdn", 0.0),
    "recsys": Workload("recsys", 32, 4, 8192, 64, 64, 4, 64, "bf16", "projected", "gdn", 0.0),
    "long": Workload("long", 1, 16, 65536, 128, 128, 2, 128, "bf16", "projected", "gdn", 0.02),
    "decode": Workload("decode", 256, 32, 1, 128, 128, 4, 64, "bf16", "projected", "gdn", 0.02,
                       steps=1000),
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _gates(g, shape, recipe):
    a_noise = torch.randn(shape, generator=g)
    b_noise = torch.randn(shape, generator=g)
    if recipe == "tiny":
        alpha = torch.exp(-0.1 * F.softplus(a_noise))
    else:
        alpha = torch.exp(-F.softplus(a_noise - 3.0))
    beta = torch.sigmoid(b_noise)
    return alpha.float().contiguous(), beta.float().contiguous()


def _projections(g, wl: Workload):
    d = wl.dk
    P_u = torch.randn((wl.H, wl.L, wl.dv, d), generator=g) / d ** 0.5
    P_w = torch.randn((wl.H, wl.L, wl.dk, d), generator=g) / d ** 0.5
    return P_u, P_w


def _project(z, P_u, P_w, L, io_dtype, rows_per_block=1 << 16):
    """u_{l} = 0.5^l P_u z and w_l = normalize(P_w z) for every token; z is [N, H, d]."""
    N, H, d = z.shape
    u = torch.empty((N, H, L, P_u.shape[2]), dtype=io_dtype)
    w = torch.empty((N, H, L, P_w.shape[2]), dtype=io_dtype)
    scale = torch.tensor([0.5 ** (l + 1) for l in range(L)]).view(1, 1, L, 1)
    for s in range(0, N, rows_per_block):
        zb = z[s:s + rows_per_block]
        ub = torch.einsum("hlvd,nhd->nhlv", P_u, zb) * scale
        wb = F.normalize(torch.einsum("hlkd,nhd->nhlk", P_w, zb), dim=-1)
        u[s:s + rows_per_block] = ub.to(io_dtype)
        w[s:s + rows_per_block] = wb.to(io_dtype)
    return u, w


def make_inputs(wl: Workload, seed: int = 0) -> dict:
    """Draw one scan-forward batch.  Returns CPU tensors:
    q, k [B,T,H,dk]; v [B,T,H,dv] or None; alpha, beta [B,T,H] fp32; u [B,T,H,L,dv] and
    w [B,T,H,L,dk] or None; S0 [B,H,dv,dk] fp32 or None."""
    g = _gen(seed)
    B, T, H, dk, dv = wl.B, wl.T, wl.H, wl.dk, wl.dv
    io = wl.torch_io
    q = torch.randn((B, T, H, dk), generator=g).to(io)
    k = F.normalize(torch.randn((B, T, H, dk), generator=g), dim=-1).to(io)
    alpha, beta = _gates(g, (B, T, H), wl.alpha_recipe)
    v = u = w = None
    if wl.write == "gdn":
        v = torch.randn((B, T, H, dv), generator=g).to(io)
    else:
        P_u, P_w = _projections(g, wl)
        z = torch.randn((B * T, H, dk), generator=g)
        u, w = _project(z, P_u, P_w, wl.L, io)
        u = u.view(B, T, H, wl.L, dv)
        w = w.view(B, T, H, wl.L, dk)
    S0 = None
    if wl.s0_std > 0:
        S0 = (torch.randn((B, H, dv, dk), generator=g) * wl.s0_std).float()
    return {"q": q, "k": k, "v": v, "alpha": alpha, "beta": beta, "u": u, "w": w, "S0": S0}


def make_producer_inputs(wl: Workload, seed: int = 0) -> dict:
    """Inputs of the write-term producer for a workload's shape (d = dk = dv, L ranks), random
    weights: x, v [B,T,H,d] ~ N(0, 1) bf16; conv [H,4,d] ~ N(0, 1/4) fp32; Wk, Wp [H,L,d,d] ~
    N(0, 1/d) bf16; beta [B,T,H,L] = sigmoid(N(0, 1)) fp32."""
    g = _gen(seed * 7919 + 17)
    B, T, H, d, L = wl.B, wl.T, wl.H, wl.dk, wl.L
    x = torch.randn((B, T, H, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, T, H, d), generator=g).to(torch.bfloat16)
    conv = (torch.randn((H, 4, d), generator=g) * 0.5).float().contiguous()
    Wk = (torch.randn((H, L, d, d), generator=g) / d ** 0.5).to(torch.bfloat16)
    Wp = (torch.randn((H, L, d, d), generator=g) / d ** 0.5).to(torch.bfloat16)
    beta = torch.sigmoid(torch.randn((B, T, H, L), generator=g)).float().contiguous()
    return {"x": x, "v": v, "conv": conv, "Wk": Wk, "Wp": Wp, "beta": beta}


def make_decode_state(wl: Workload, seed: int = 0) -> dict:
    """Entry state and the fixed write projections of a decode run."""
    g = _gen(seed * 1_000_003 + 7)
    S0 = (torch.randn((wl.B, wl.H, wl.dv, wl.dk), generator=g) * wl.s0_std).float()
    P_u, P_w = _projections(g, wl)
    return {"S0": S0, "P_u": P_u, "P_w": P_w}


def make_decode_step(wl: Workload, state: dict, step: int, seed: int = 0) -> dict:
    """Inputs of one single-token decode step, shaped as a T == 1 batch: q, k [B,1,H,dk];
    alpha, beta [B,1,H]; u [B,1,H,L,dv]; w [B,1,H,L,dk] (v absent).  Each step draws from its
    own seed, so any step can be regenerated without the ones before it."""
    g = _gen(seed * 1_000_003 + 1009 * (step + 1))
    B, H, dk = wl.B, wl.H, wl.dk
    io = wl.torch_io
    q = torch.randn((B, 1, H, dk), generator=g).to(io)
    k = F.normalize(torch.randn((B, 1, H, dk), generator=g), dim=-1).to(io)
    alpha, beta = _gates(g, (B, 1, H), wl.alpha_recipe)
    z = torch.randn((B, H, dk), generator=g)
    u, w = _project(z, state["P_u"], state["P_w"], wl.L, io)
    return {"q": q, "k": k, "v": None, "alpha": alpha, "beta": beta,
            "u": u.view(B, 1, H, wl.L, wl.dv), "w": w.view(B, 1, H, wl.L, dk)}


def select_heads(inputs: dict, heads) -> dict:
    """Copy out the listed (b, h) pairs as a B'=len(heads), H'=1 batch (for sampled checks)."""
    out = {}
    for key, x in inputs.items():
        if x is None:
            out[key] = None
            continue
        parts = []
        for b, h in heads:
            if key == "S0":
                parts.append(x[b:b + 1, h:h + 1])
            else:
                parts.append(x[b:b + 1, :, h:h + 1])
        out[key] = torch.cat(parts, dim=0).contiguous()
    return out
