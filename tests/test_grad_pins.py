"""Pins of the backward-pass oracle (oracle/scan_grad.py): every gradient against central finite
differences of the forward oracle (oracle.scan_ref, the C implementation), for the GDN write and
the rank-L write, with an entry state and an exit-state gradient.  Planted mistakes are caught."""
import numpy as np
import pytest
import torch

import oracle
from oracle.scan_grad import scan_grad_ref


def _case(seed, gdn, B=1, T=5, H=2, dk=3, dv=2, L=2):
    g = torch.Generator().manual_seed(seed)
    k = torch.nn.functional.normalize(torch.randn((B, T, H, dk), generator=g), dim=-1)
    c = dict(
        q=torch.randn((B, T, H, dk), generator=g),
        k=k,
        alpha=torch.rand((B, T, H), generator=g) * 0.3 + 0.65,
        beta=torch.rand((B, T, H), generator=g) * 0.8 + 0.1,
        S0=torch.randn((B, H, dv, dk), generator=g) * 0.5,
    )
    if gdn:
        c.update(v=torch.randn((B, T, H, dv), generator=g), u=None, w=None)
    else:
        c.update(v=None, u=torch.randn((B, T, H, L, dv), generator=g) * 0.5,
                 w=torch.randn((B, T, H, L, dk), generator=g) * 0.5)
    up = dict(do=torch.randn((B, T, H, dv), generator=g).double(),
              dS=torch.randn((B, H, dv, dk), generator=g).double())
    return {n: (None if t is None else t.float().contiguous()) for n, t in c.items()}, up


def _loss(c, up):
    o, S = oracle.scan_ref(c["q"], c["k"], c["v"], c["alpha"], c["beta"], c["u"], c["w"], c["S0"])
    return float(np.sum(up["do"].numpy() * o) + np.sum(up["dS"].numpy() * S))


def _fd(c, up, name, h=1e-3):
    """Central differences in every element of input `name` (fp32 inputs: the step actually
    taken is measured, not assumed)."""
    x = c[name]
    grad = np.zeros(x.shape)
    flat = x.view(-1)
    for i in range(flat.numel()):
        x0 = float(flat[i])
        xp, xm = np.float32(x0 + h * max(1.0, abs(x0))), np.float32(x0 - h * max(1.0, abs(x0)))
        flat[i] = float(xp)
        lp = _loss(c, up)
        flat[i] = float(xm)
        lm = _loss(c, up)
        flat[i] = x0
        grad.reshape(-1)[i] = (lp - lm) / (float(xp) - float(xm))
    return grad


def _check(gdn, grads_fn):
    c, up = _case(3 if gdn else 4, gdn)
    got = grads_fn(c, up)
    names = ["q", "k", "alpha", "beta", "S0"] + (["v"] if gdn else ["u", "w"])
    for n in names:
        np.testing.assert_allclose(got["d" + n], _fd(c, up, n), rtol=1e-5, atol=1e-6, err_msg=n)


def _oracle_grads(mutant=0):
    def run(c, up):
        return scan_grad_ref(c["q"], c["k"], c["v"], c["alpha"], c["beta"], c["u"], c["w"], c["S0"],
                             do=up["do"], dS_final=up["dS"], mutant=mutant)
    return run


@pytest.mark.parametrize("gdn", [True, False], ids=["gdn_write", "rank_L_write"])
def test_gradients_match_finite_differences(gdn):
    _check(gdn, _oracle_grads())


@pytest.mark.parametrize("mutant", [1, 2, 3])
def test_planted_mistakes_are_caught(mutant):
    with pytest.raises(AssertionError):
        _check(False, _oracle_grads(mutant))
