"""Randomised shapes (hypothesis) for the two numpy mirrors of the chunked design against the fp64
oracles: the chunked forward (tests/chunk_algebra.py) and the chunked backward
(tests/chunk_backward.py), over ragged token counts, chunk sizes that do and do not divide T,
both write forms, small widths and ranks."""
import numpy as np
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from oracle.scan_grad import scan_grad_ref
from tests.chunk_algebra import chunked_forward
from tests.chunk_backward import chunked_backward


def _case(seed, T, H, dk, dv, L, gdn):
    g = torch.Generator().manual_seed(seed)
    c = dict(
        q=torch.randn((1, T, H, dk), generator=g),
        k=torch.nn.functional.normalize(torch.randn((1, T, H, dk), generator=g), dim=-1),
        alpha=torch.rand((1, T, H), generator=g) * 0.4 + 0.55,
        beta=torch.rand((1, T, H), generator=g) * 0.9 + 0.05,
        S0=torch.randn((1, H, dv, dk), generator=g) * 0.3,
    )
    if gdn:
        c.update(v=torch.randn((1, T, H, dv), generator=g), u=None, w=None)
    else:
        c.update(v=None, u=torch.randn((1, T, H, L, dv), generator=g) * 0.5,
                 w=torch.randn((1, T, H, L, dk), generator=g) * 0.5)
    return {n: (None if t is None else t.float().contiguous()) for n, t in c.items()}


shapes = dict(seed=st.integers(0, 10_000), T=st.integers(1, 40), H=st.integers(1, 2),
              dk=st.integers(1, 5), dv=st.integers(1, 5), L=st.integers(1, 3), gdn=st.booleans(),
              chunk=st.sampled_from([1, 2, 3, 5, 8, 16, 64]))


@settings(max_examples=40, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(**shapes)
def test_chunked_forward_matches_oracle(seed, T, H, dk, dv, L, gdn, chunk):
    x = _case(seed, T, H, dk, dv, L, gdn)
    o_ref, S_ref = oracle.scan_ref(**x)
    o, S = chunked_forward(**x, chunk=chunk)
    np.testing.assert_allclose(o, o_ref, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(S, S_ref, rtol=1e-9, atol=1e-9)


@settings(max_examples=25, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(**shapes)
def test_chunked_backward_matches_oracle(seed, T, H, dk, dv, L, gdn, chunk):
    x = _case(seed, T, H, dk, dv, L, gdn)
    g = torch.Generator().manual_seed(seed + 1)
    up = dict(do=torch.randn((1, T, H, dv), generator=g).double(),
              dS_final=torch.randn((1, H, dv, dk), generator=g).double())
    ref = scan_grad_ref(**x, **up)
    got = chunked_backward(**x, **up, chunk=chunk)
    for n in ("dq", "dk", "dalpha", "dbeta", "dS0") + (("dv",) if gdn else ("du", "dw")):
        np.testing.assert_allclose(got[n], ref[n], rtol=1e-8, atol=1e-9, err_msg=n)
