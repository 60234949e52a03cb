"""The chunked backward design (tests/chunk_backward.py) against the token-level backward oracle:
the reverse chunk recurrence dS_c = dS_{c+1} E_c^T + dO_c^T Qt_c gives the state gradient at
every chunk boundary, and per-chunk backward passes from those boundaries give every input
gradient, for several chunk sizes and both write forms."""
import numpy as np
import pytest
import torch

from oracle.scan_grad import scan_grad_ref
from tests.chunk_backward import chunked_backward


def _case(seed, gdn, B=1, T=23, H=2, dk=4, dv=3, L=2):
    g = torch.Generator().manual_seed(seed)
    c = dict(
        q=torch.randn((B, T, H, dk), generator=g).double(),
        k=torch.nn.functional.normalize(torch.randn((B, T, H, dk), generator=g), dim=-1).double(),
        alpha=(torch.rand((B, T, H), generator=g) * 0.3 + 0.65).double(),
        beta=(torch.rand((B, T, H), generator=g) * 0.8 + 0.1).double(),
        S0=(torch.randn((B, H, dv, dk), generator=g) * 0.5).double(),
    )
    if gdn:
        c.update(v=torch.randn((B, T, H, dv), generator=g).double(), u=None, w=None)
    else:
        c.update(v=None, u=(torch.randn((B, T, H, L, dv), generator=g) * 0.5).double(),
                 w=(torch.randn((B, T, H, L, dk), generator=g) * 0.5).double())
    c["do"] = torch.randn((B, T, H, dv), generator=g).double()
    c["dS_final"] = torch.randn((B, H, dv, dk), generator=g).double()
    return c


@pytest.mark.parametrize("gdn", [True, False], ids=["gdn_write", "rank_L_write"])
@pytest.mark.parametrize("chunk", [1, 3, 8, 16, 64])
def test_chunked_backward_equals_token_backward(gdn, chunk):
    c = _case(7 + chunk, gdn)
    ref = scan_grad_ref(**c)
    got = chunked_backward(**c, chunk=chunk)
    for n in ("dq", "dk", "dalpha", "dbeta", "dS0") + (("dv",) if gdn else ("du", "dw")):
        np.testing.assert_allclose(got[n], ref[n], rtol=1e-9, atol=1e-10, err_msg=n)
