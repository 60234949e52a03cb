"""Pins of the write-term producer's fp64 oracle (``oracle/write_producer.py``) against what the
mathematics fixes independently of it: special cases that reduce to a library routine (a causal
depthwise convolution, a matrix product, the exact GELU), the telescoping of the residual chain,
the zero-gain case, linearity in the gate, and a hand-worked case.  Every planted mistake in
``write_producer_ref(mutant=...)`` fails at least one of them."""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle.write_producer import CONV_WIDTH, gelu, write_producer_ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_producer_d1.json")


def _case(seed, B=1, T=9, H=2, d=4, L=3):
    g = torch.Generator().manual_seed(seed)
    return dict(
        x=torch.randn((B, T, H, d), generator=g),
        v=torch.randn((B, T, H, d), generator=g),
        conv=torch.randn((H, CONV_WIDTH, d), generator=g) / 2,
        Wk=torch.randn((H, L, d, d), generator=g) / d ** 0.5,
        Wp=torch.randn((H, L, d, d), generator=g) / d ** 0.5,
        beta=torch.rand((B, T, H, L), generator=g) * 0.9 + 0.1,
    )


def _anchor_by_conv1d(x, conv):
    """Causal depthwise convolution by torch's conv1d: out_t = sum_j c_j x_{t-j}."""
    B, T, H, d = x.shape
    out = torch.empty((B, T, H, d), dtype=torch.float64)
    for h in range(H):
        weight = conv[h].double().flip(0).t().unsqueeze(1)          # [d, 1, width]
        seq = x[:, :, h].double().transpose(1, 2)                    # [B, d, T]
        y = F.conv1d(F.pad(seq, (CONV_WIDTH - 1, 0)), weight, groups=d)
        out[:, :, h] = y.transpose(1, 2)
    return out.numpy()


def pin_anchor(run):
    """W_k = I and W_p = 0: the directions are the anchor itself."""
    c = _case(1)
    d, L = c["x"].shape[-1], c["Wk"].shape[1]
    c["Wk"] = torch.eye(d).expand(c["Wk"].shape[0], L, d, d).clone()
    c["Wp"] = torch.zeros_like(c["Wp"])
    _, w, _ = run(**c)
    a = _anchor_by_conv1d(c["x"], c["conv"])
    for l in range(L):
        np.testing.assert_allclose(w[:, :, :, l], a, rtol=1e-12, atol=1e-12)


def pin_directions(run):
    """Anchor = x (c = [1, 0, 0, 0]): the directions are W_k^(l) x by a library matmul."""
    c = _case(2)
    c["conv"] = torch.zeros_like(c["conv"])
    c["conv"][:, 0] = 1.0
    _, w, _ = run(**c)
    ref = torch.einsum("hlij,bthj->bthli", c["Wk"].double(), c["x"].double()).numpy()
    np.testing.assert_allclose(w, ref, rtol=1e-12, atol=1e-12)


def pin_gelu_step(run):
    """L = 1, W_p = I, anchor = x: delta = GELU(x * v), by torch's exact GELU."""
    c = _case(3, L=1)
    d = c["x"].shape[-1]
    c["conv"] = torch.zeros_like(c["conv"])
    c["conv"][:, 0] = 1.0
    c["Wp"] = torch.eye(d).expand(c["Wp"].shape[0], 1, d, d).clone()
    u, _, r = run(**c)
    delta = F.gelu(c["x"].double() * c["v"].double(), approximate="none").numpy()
    np.testing.assert_allclose(u[:, :, :, 0], c["beta"].double().numpy()[..., 0:1] * delta,
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r, c["v"].double().numpy() - delta, rtol=1e-12, atol=1e-12)


def pin_telescoping(run):
    """The residual chain telescopes: sum_l delta^(l) + r^(L+1) = v, delta^(l) = u_l / beta_l."""
    c = _case(4, L=4)
    u, _, r = run(**c)
    deltas = u / c["beta"].double().numpy()[..., None]
    np.testing.assert_allclose(deltas.sum(axis=3) + r, c["v"].double().numpy(), rtol=1e-12,
                               atol=1e-12)
    assert np.abs(deltas).max() > 1e-3  # the chain did something


def pin_zero_gain(run):
    """W_p = 0: every delta is GELU(0) = 0, nothing is written and the residual stays v."""
    c = _case(5)
    c["Wp"] = torch.zeros_like(c["Wp"])
    u, _, r = run(**c)
    assert np.abs(u).max() == 0.0
    np.testing.assert_array_equal(r, c["v"].double().numpy())


def pin_gate_linearity(run):
    """The gate scales the written values only: u is linear in beta, w and r do not move."""
    c = _case(6)
    u1, w1, r1 = run(**c)
    c2 = dict(c, beta=c["beta"].double() * 3.0)  # exact: 3 x an fp32 value fits in fp64
    u2, w2, r2 = run(**c2)
    np.testing.assert_allclose(u2, 3.0 * u1, rtol=1e-12, atol=1e-14)
    np.testing.assert_array_equal(w1, w2)
    np.testing.assert_array_equal(r1, r2)


def pin_hand_worked(run):
    """d = 1, L = 2, T = 3, one head, worked step by step in plain arithmetic (first GELU
    arguments 1, 1, -2; tests/golden/hand_worked_producer_d1.json holds the derivation, written by
    tests/golden/make_hand_worked_producer.py without calling the oracle)."""
    with open(GOLDEN) as f:
        g = json.load(f)
    t = lambda a: torch.tensor(a, dtype=torch.float64)
    u, w, r = run(x=t(g["x"]), v=t(g["v"]), conv=t(g["conv"]), Wk=t(g["Wk"]), Wp=t(g["Wp"]),
                  beta=t(g["beta"]))
    np.testing.assert_allclose(u, np.array(g["u"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(w, np.array(g["w"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(r, np.array(g["r_final"]), rtol=0, atol=1e-12)


PINS = [pin_anchor, pin_directions, pin_gelu_step, pin_telescoping, pin_zero_gain,
        pin_gate_linearity, pin_hand_worked]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_meets_pin(pin):
    pin(write_producer_ref)


def test_gelu_known_values():
    # Phi(1) = 0.841344746068543 (standard normal table); GELU(x) = x Phi(x)
    assert gelu(1.0) == pytest.approx(0.8413447460685429, abs=1e-15)
    assert gelu(-1.0) == pytest.approx(-0.15865525393145707, abs=1e-15)
    assert gelu(0.0) == 0.0
    for z in (-3.0, -0.5, 0.25, 2.0):
        assert gelu(z) == pytest.approx(F.gelu(torch.tensor(z, dtype=torch.float64)).item(), abs=1e-15)


@pytest.mark.parametrize("mutant", [1, 2, 3, 4, 5, 6])
def test_every_planted_mistake_fails_a_pin(mutant):
    def run(**kw):
        return write_producer_ref(**kw, mutant=mutant)

    caught = 0
    for pin in PINS:
        try:
            pin(run)
        except AssertionError:
            caught += 1
    assert caught >= 1, f"mutant {mutant} passed every pin"


def test_hand_worked_golden_is_consistent_with_its_derivation():
    """The golden file's numbers follow from its own stated intermediate values (anchors, GELU
    arguments), independently of the oracle."""
    with open(GOLDEN) as f:
        g = json.load(f)
    phi = lambda z: 0.5 * (1.0 + math.erf(z / math.sqrt(2.0)))
    for t, step in enumerate(g["derivation"]):
        for l, arg in enumerate(step["gelu_args"]):
            expect = arg * phi(arg)
            assert step["deltas"][l] == pytest.approx(expect, abs=1e-12)
