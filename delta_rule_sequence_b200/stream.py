"""Streaming chunk-level inference with an online binary counter over chunk elements.

"Sequential Parallel Duality in Prefix Scannable Models" (papernotes), key design 3 and the worked
example: at inference time the history is kept as at most one complete subtree root per slot k
(a summary of 2^k chunks); a new chunk is inserted like a binary increment (while slot k is full,
merge its root with the carry, older on the left, and carry into slot k + 1), and the prefix
state is the fold of the non-empty roots from the highest slot (oldest) to the lowest (newest).
The roots then cut the history into power-of-two blocks merged in the same bracketing as the
static Blelloch up-sweep, with at most ceil(log2(n + 1)) roots after n chunks and one merge per
trailing one of the chunk count.

Here the elements are the scan's affine chunk elements (E, f) (the map S -> S E + f of a token
segment; key design 2), so every bracketing gives the same state: the counter serves as the
streaming decode path and as a check of the fixed-bracketing view.  Per chunk, the outputs come
from the chunk's scan forward started at the prefix state (the pages' Inf(s_{i-1}, C_i)).

The element, composition and fold are parameters so that the bookkeeping can be checked on CPU
with reference implementations; they default to the library's kernels
(``prism_scan_segment_element``, and ``prism_state_fold`` for both S E + f and the composition
(E_a, f_a) then (E_b, f_b) = (E_a E_b, f_a E_b + f_b)).
"""
from __future__ import annotations


def _library_steps():
    from delta_rule_sequence_b200 import prism

    def element(q, k, v, alpha, beta, u, w, chunk):
        return prism.prism_scan_segment_element(q, k, v, alpha, beta, u, w, chunk=chunk)

    def compose(older, newer):  # (E_a, f_a) then (E_b, f_b) = (E_a E_b, f_a E_b + f_b)
        (Ea, fa), (Eb, fb) = older, newer
        return prism.prism_state_fold(Ea, Eb, _zeros_like(Ea)), prism.prism_state_fold(fa, Eb, fb)

    def fold(S, E, f):
        return prism.prism_state_fold(S, E, f)

    def scan(q, k, v, alpha, beta, u, w, S0, chunk):
        return prism.prism_scan_fwd(q, k, v, alpha, beta, u, w, S0, chunk=chunk)

    return element, compose, fold, scan


def _zeros_like(t):
    import torch

    return torch.zeros_like(t)


class ChunkCounter:
    """Online binary counter of chunk elements (see the module docstring)."""

    def __init__(self, compose_fn, fold_fn):
        self.compose, self.fold = compose_fn, fold_fn
        self.roots = []     # roots[k]: the element of 2^k consecutive chunks, or None
        self.count = 0      # chunks pushed
        self.merges = 0     # compositions performed so far

    def push(self, element):
        k = 0
        while k < len(self.roots) and self.roots[k] is not None:
            element = self.compose(self.roots[k], element)  # the older block on the left
            self.roots[k] = None
            self.merges += 1
            k += 1
        if k == len(self.roots):
            self.roots.append(None)
        self.roots[k] = element
        self.count += 1

    def live_roots(self):
        """(slot, element) of the non-empty slots, highest (oldest history) first."""
        return [(k, self.roots[k]) for k in reversed(range(len(self.roots))) if self.roots[k] is not None]

    def state(self, S0=None):
        """The prefix state: the entry state carried through every root, oldest first."""
        S = S0
        for _, (E, f) in self.live_roots():
            S = self.fold(S, E, f)
        return S


class StreamingScan:
    """Chunk-by-chunk inference: outputs of each arriving chunk from the current prefix state,
    then the chunk's element pushed into the counter.  Inputs per chunk as for prism_scan_fwd
    ([B, c, H, ...] device tensors of the chunk's tokens); S0 the state before the stream."""

    def __init__(self, S0=None, *, chunk=64, element_fn=None, compose_fn=None, fold_fn=None,
                 scan_fn=None):
        if None in (element_fn, compose_fn, fold_fn, scan_fn):
            e, c, f, s = _library_steps()
            element_fn, compose_fn, fold_fn, scan_fn = (element_fn or e, compose_fn or c,
                                                        fold_fn or f, scan_fn or s)
        self.element, self.scan, self.chunk = element_fn, scan_fn, chunk
        self.S0 = S0
        self.counter = ChunkCounter(compose_fn, fold_fn)

    def step(self, q, k, v, alpha, beta, u=None, w=None):
        """Process one chunk: returns its outputs o [B, c, H, dv]."""
        entry = self.counter.state(self.S0)
        o, _ = self.scan(q, k, v, alpha, beta, u, w, entry, self.chunk)
        self.counter.push(self.element(q, k, v, alpha, beta, u, w, self.chunk))
        return o

    def state(self):
        """The state after every chunk so far."""
        return self.counter.state(self.S0)
