"""Shared helpers of the GPU parity tests: run the CUDA path and the fp64 oracle on the same seeded
bytes and compare element by element.

Tolerance (bf16 I/O 2e-2, fp32 I/O 1e-4): an element passes iff |x - r| <= tol * (1 + |r|),
for o and S_final alike."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from delta_rule_sequence_b200.workloads import select_heads

TOL = {"bf16": 2e-2, "f32": 1e-4}


def to_device(inputs, device="cuda"):
    return {n: (None if x is None else x.to(device)) for n, x in inputs.items()}


def compare(name, got, ref, tol):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{name}: non-finite values from the CUDA path"
    err = np.abs(got - ref)
    bound = tol * (1.0 + np.abs(ref))
    bad = err > bound
    max_abs = float(err.max()) if err.size else 0.0
    if bad.any():
        idx = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(
            f"{name}: {int(bad.sum())}/{bad.size} elements out of tolerance {tol}; worst at {idx}: "
            f"got {got[idx]!r} ref {ref[idx]!r}; max abs err {max_abs:.3e}")
    return max_abs


def run_cuda_scan(dev_inputs, chunk):
    from delta_rule_sequence_b200.prism import prism_scan_fwd

    x = dev_inputs
    o, Sf = prism_scan_fwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["u"], x["w"],
                           x["S0"], chunk=chunk)
    torch.cuda.synchronize()
    return o, Sf


def check_scan_full(inputs, chunk, io):
    """Every element of o and S_final against the oracle."""
    o, Sf = run_cuda_scan(to_device(inputs), chunk)
    o_ref, S_ref = oracle.scan_ref(**inputs)
    tol = TOL[io]
    return (compare("o", o.float().cpu().numpy(), o_ref, tol),
            compare("S_final", Sf.cpu().numpy(), S_ref, tol))


def check_scan_sampled(inputs, chunk, io, heads):
    """Full-size launch; the listed (b, h) sequences are checked against the oracle."""
    o, Sf = run_cuda_scan(to_device(inputs), chunk)
    sub = select_heads(inputs, heads)
    o_ref, S_ref = oracle.scan_ref(**sub)
    o_got = torch.cat([o[b:b + 1, :, h:h + 1].cpu() for b, h in heads], 0).float().numpy()
    S_got = torch.cat([Sf[b:b + 1, h:h + 1].cpu() for b, h in heads], 0).numpy()
    tol = TOL[io]
    return compare("o", o_got, o_ref, tol), compare("S_final", S_got, S_ref, tol)
