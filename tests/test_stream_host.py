"""The online binary counter of delta_rule_sequence_b200.stream on CPU: its roots reproduce the
static Blelloch up-sweep's bracketing (checked with symbolic elements that record how they were
merged), the counts the pages state (at most ceil(log2(n + 1)) roots, one merge per trailing one),
and chunk-by-chunk streaming inference equal to one pass of the fp64 oracle, with the oracle in
place of the kernels (the kernels are checked on the GPU)."""
import math

import numpy as np
import pytest
import torch

from delta_rule_sequence_b200.stream import ChunkCounter, StreamingScan


def _block(lo, size):
    """The static Blelloch up-sweep's subtree over chunks lo .. lo + size - 1 (size a power of 2)."""
    if size == 1:
        return f"x{lo}"
    h = size // 2
    return f"({_block(lo, h)}+{_block(lo + h, h)})"


@pytest.mark.parametrize("n", list(range(1, 40)))
def test_counter_roots_are_the_blelloch_subtrees(n):
    counter = ChunkCounter(lambda a, b: (f"({a[0]}+{b[0]})",) * 2, lambda S, E, f: S + [E])
    merges_per_push = []
    for i in range(n):
        before = counter.merges
        counter.push((f"x{i}", f"x{i}"))
        merges_per_push.append(counter.merges - before)
        # one merge per trailing one of the count before this push
        c, t = i, 0
        while c & 1:
            c >>= 1
            t += 1
        assert merges_per_push[-1] == t
    # the roots, oldest first, are the power-of-two blocks of n's binary expansion
    expect, lo = [], 0
    for k in reversed(range(n.bit_length())):
        if n >> k & 1:
            expect.append(_block(lo, 1 << k))
            lo += 1 << k
    assert [E for _, (E, _) in counter.live_roots()] == expect
    assert counter.state([]) == expect
    assert len(expect) == bin(n).count("1") <= math.ceil(math.log2(n + 1))
    assert counter.merges == n - bin(n).count("1")


def _oracle_steps():
    import oracle

    def element(q, k, v, a, b, u, w, chunk):
        B, T, H, dk = q.shape
        eye = np.broadcast_to(np.eye(dk), (B, H, dk, dk)).copy()
        if u is None:
            _, E = oracle.scan_ref(q, k, torch.zeros_like(v), a, b, S0=eye, n_threads=1)
        else:
            _, E = oracle.scan_ref(q, k, None, a, b, torch.zeros_like(u), w, S0=eye, n_threads=1)
        _, f = oracle.scan_ref(q, k, v, a, b, u, w, None, n_threads=1)
        return torch.from_numpy(E), torch.from_numpy(f)

    def compose(older, newer):
        (Ea, fa), (Eb, fb) = older, newer
        return Ea @ Eb, fa @ Eb + fb

    def fold(S, E, f):
        return f.clone() if S is None else S.double() @ E + f

    def scan(q, k, v, a, b, u, w, S0, chunk):
        o, Sf = oracle.scan_ref(q, k, v, a, b, u, w, S0, n_threads=1)
        return torch.from_numpy(o), torch.from_numpy(Sf)

    return element, compose, fold, scan


@pytest.mark.parametrize("name,over,c", [
    ("tiny", dict(T=7 * 32, s0_std=0.05), 32),                                   # GDN write
    ("long", dict(H=1, T=5 * 16, dk=16, dv=16, io="f32", L=2), 16),             # rank-L write
])
def test_streaming_equals_one_pass(name, over, c):
    import oracle
    from delta_rule_sequence_b200.workloads import WORKLOADS, make_inputs

    wl = WORKLOADS[name].with_(**over)
    x = make_inputs(wl, seed=13)
    element, compose, fold, scan = _oracle_steps()
    s = StreamingScan(x["S0"], chunk=c, element_fn=element, compose_fn=compose, fold_fn=fold,
                      scan_fn=scan)
    outs = []
    for t0 in range(0, wl.T, c):
        part = {n: (None if t is None or n == "S0" else t[:, t0:t0 + c].contiguous()) for n, t in x.items()}
        outs.append(s.step(part["q"], part["k"], part["v"], part["alpha"], part["beta"], part["u"],
                           part["w"]).numpy())
    o_ref, S_ref = oracle.scan_ref(**x)
    np.testing.assert_allclose(np.concatenate(outs, axis=1), o_ref, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(s.state().numpy(), S_ref, rtol=1e-10, atol=1e-10)
    assert s.counter.count == wl.T // c
