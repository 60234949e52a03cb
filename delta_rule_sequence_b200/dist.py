"""One process per GPU: the host side of running the scan on several devices.

Two ways to spread the work, both over ``torch.distributed`` (NCCL between GPUs; the same calls
run on gloo between CPU processes, which is how the tests exercise them):

* Weak scaling over independent sequences.  The B*H (batch, head) sequences of a layer do not
  interact, so each rank processes its own share with no collective in the data path; only the
  timing (a device-side max over ranks) crosses ranks.
* Context parallelism along T, for few long sequences.  Rank r holds the r-th contiguous token
  segment.  It encodes its segment as the affine map S -> S E_r + f_r (the segment element of
  "Sequential Parallel Duality in Prefix Scannable Models", method overview: elements of an
  associative operator compose in order), the ranks all-gather the elements (one exchange of
  2 * B*H * d^2 fp32 per rank), each rank folds the elements of the ranks before it into its entry
  state, and then runs the ordinary scan forward on its segment from that state.  The exit state
  of the whole sequence is the last rank's exit state.

The compute steps are the library's kernels (``prism_scan_segment_element``, ``prism_state_fold``,
``prism_scan_fwd``); they are parameters of ``cp_scan_fwd`` so that the exchange can be checked
on CPU processes with reference implementations in their place.
"""
from __future__ import annotations

import os
from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class RankInfo:
    rank: int
    world: int
    local_rank: int


def rank_info() -> RankInfo:
    """Rank, world size and local rank from the launcher's environment (1 process: 0, 1, 0)."""
    return RankInfo(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float, device=None) -> float:
    """The largest `x` over all ranks (a time, so that a job is as slow as its slowest rank).
    Without an initialised process group this is `x`."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_range(n: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous share [lo, hi) of n items for `rank` of `world`; the first n % world ranks get
    one more item than the others."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError(f"shard_range: bad arguments n={n} rank={rank} world={world}")
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def weak_scaling_value(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: the units every rank processed, over the slowest rank's time."""
    if max_seconds <= 0:
        raise ValueError("weak_scaling_value: the time must be positive")
    return world * units_per_rank / max_seconds


def _all_gather(t: torch.Tensor, world: int) -> list[torch.Tensor]:
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous())
    return parts


def cp_scan_fwd(q, k, v, alpha, beta, u=None, w=None, S0=None, *, chunk=64,
                element_fn=None, fold_fn=None, scan_fn=None):
    """Context-parallel scan forward.  Every rank passes its own contiguous token segment of the
    same sequences ([B, T_r, H, ...], in rank order) and the same S0; returns this rank's outputs
    and the exit state of the whole sequence (identical on every rank).

    element_fn(q, k, v, alpha, beta, u, w, chunk) -> (E, f);  fold_fn(S, E, f) -> S E + f (S may
    be None for zero);  scan_fn(q, k, v, alpha, beta, u, w, S0, chunk) -> (o, S_final).  They
    default to the library's kernels (device tensors).
    """
    if element_fn is None or fold_fn is None or scan_fn is None:
        from delta_rule_sequence_b200 import prism

        if element_fn is None:
            def element_fn(q_, k_, v_, a_, b_, u_, w_, c_):
                return prism.prism_scan_segment_element(q_, k_, v_, a_, b_, u_, w_, chunk=c_)
        if fold_fn is None:
            def fold_fn(S_, E_, f_):
                return prism.prism_state_fold(S_, E_, f_)
        if scan_fn is None:
            def scan_fn(q_, k_, v_, a_, b_, u_, w_, S0_, c_):
                return prism.prism_scan_fwd(q_, k_, v_, a_, b_, u_, w_, S0_, chunk=c_)
    world = dist.get_world_size() if dist.is_initialized() else 1
    rank = dist.get_rank() if dist.is_initialized() else 0
    if world == 1:
        return scan_fn(q, k, v, alpha, beta, u, w, S0, chunk)
    # 1. this segment's element, 2. one exchange, 3. the fold of the elements before this rank
    E, f = element_fn(q, k, v, alpha, beta, u, w, chunk)
    Es, fs = _all_gather(E, world), _all_gather(f, world)
    entry = S0
    for j in range(rank):
        entry = fold_fn(entry, Es[j], fs[j])
    # 4. the ordinary forward from the entry state; the last rank's exit state is the sequence's
    o, S_last = scan_fn(q, k, v, alpha, beta, u, w, entry, chunk)
    S_final = S_last.contiguous() if rank == world - 1 else torch.empty_like(fs[0])
    dist.broadcast(S_final, src=world - 1)
    return o, S_final
