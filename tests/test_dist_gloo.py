"""The multi-process host logic on CPU: two gloo ranks (world size 2) exercise the device-side
max over ranks, the sharding and throughput arithmetic of weak scaling, and the exchange of the
context-parallel scan, whose compute steps are supplied by the fp64 oracle here (the kernels are
checked against the same oracle on the GPU)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from delta_rule_sequence_b200 import dist as pdist


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(fn, world=2, *args):
    import queue as _queue

    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(fn, r, world, port, q, args)) for r in range(world)]
    for p in procs:
        p.start()
    results = []
    try:
        for _ in range(world):  # drain before joining: a large result blocks its sender otherwise
            results.append(q.get(timeout=180))
    except _queue.Empty:
        pass
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
            pytest.fail("a gloo rank did not finish")
        assert p.exitcode == 0, f"rank exited with {p.exitcode}"
    assert len(results) == world
    return sorted(results, key=lambda r: r[0])


def _worker(fn, rank, world, port, q, args):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        q.put((rank, fn(rank, world, *args)))
    finally:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------------------------------------

def _max_case(rank, world):
    info = pdist.rank_info()
    assert (info.rank, info.world) == (rank, world)
    return pdist.max_over_ranks(1.5 + rank)


def test_max_over_ranks_two_gloo_ranks():
    res = _run(_max_case)
    assert [r[1] for r in res] == [2.5, 2.5]


def test_max_over_ranks_without_group():
    assert pdist.max_over_ranks(3.25) == 3.25


@pytest.mark.parametrize("n,world", [(0, 2), (7, 2), (32, 8), (5, 8), (1, 1)])
def test_shard_range_covers_everything_once(n, world):
    seen = []
    for r in range(world):
        lo, hi = pdist.shard_range(n, r, world)
        assert 0 <= lo <= hi <= n
        seen.extend(range(lo, hi))
    assert seen == list(range(n))


def test_shard_range_rejects_bad_arguments():
    with pytest.raises(ValueError):
        pdist.shard_range(4, 2, 2)


def test_weak_scaling_value():
    assert pdist.weak_scaling_value(16384, 4, 0.002) == pytest.approx(4 * 16384 / 0.002)
    with pytest.raises(ValueError):
        pdist.weak_scaling_value(1, 1, 0.0)


# ---------------------------------------------------------------------------------------------
# context parallelism: each rank owns a contiguous token segment

def _oracle_steps():
    import oracle

    def element(q, k, v, a, b, u, w, chunk):
        B, T, H, dk = q.shape
        eye = np.broadcast_to(np.eye(dk), (B, H, dk, dk)).copy()
        if u is None:   # the write off: v = 0
            _, E = oracle.scan_ref(q, k, torch.zeros_like(v), a, b, S0=eye, n_threads=1)
        else:
            _, E = oracle.scan_ref(q, k, None, a, b, torch.zeros_like(u), w, S0=eye, n_threads=1)
        _, f = oracle.scan_ref(q, k, v, a, b, u, w, None, n_threads=1)
        return torch.from_numpy(E), torch.from_numpy(f)

    def fold(S, E, f):
        return f.clone() if S is None else torch.matmul(S.double(), E) + f

    def scan(q, k, v, a, b, u, w, S0, chunk):
        o, Sf = oracle.scan_ref(q, k, v, a, b, u, w, S0, n_threads=1)
        return torch.from_numpy(o), torch.from_numpy(Sf)

    return element, fold, scan


def _cp_case(rank, world, name, over, cuts):
    from delta_rule_sequence_b200.workloads import WORKLOADS, make_inputs

    wl = WORKLOADS[name].with_(**over)
    x = make_inputs(wl, seed=11)
    lo, hi = cuts[rank], cuts[rank + 1]
    seg = {n: (None if t is None or n == "S0" else t[:, lo:hi].contiguous()) for n, t in x.items()}
    element, fold, scan = _oracle_steps()
    o, S = pdist.cp_scan_fwd(seg["q"], seg["k"], seg["v"], seg["alpha"], seg["beta"], seg["u"],
                             seg["w"], x["S0"], chunk=wl.chunk, element_fn=element, fold_fn=fold,
                             scan_fn=scan)
    return o.numpy(), S.numpy(), lo, hi


@pytest.mark.parametrize("name,over,cuts", [
    ("tiny", dict(T=192, s0_std=0.05), [0, 96, 192]),        # Gated-DeltaNet write, ragged chunks
    ("long", dict(H=1, T=160, dk=32, dv=32, io="f32"), [0, 64, 160]),  # rank-L write, nonzero S0
])
def test_context_parallel_two_ranks_match_one_pass(name, over, cuts):
    import oracle
    from delta_rule_sequence_b200.workloads import WORKLOADS, make_inputs

    res = _run(_cp_case, 2, name, over, cuts)
    wl = WORKLOADS[name].with_(**over)
    o_ref, S_ref = oracle.scan_ref(**make_inputs(wl, seed=11))
    for _, (o, S, lo, hi) in res:
        np.testing.assert_allclose(o, o_ref[:, lo:hi], rtol=1e-10, atol=1e-10)
        np.testing.assert_allclose(S, S_ref, rtol=1e-10, atol=1e-10)


def test_context_parallel_catches_a_wrong_fold_order():
    """The exchange is sensitive to the order the elements are folded in: folding rank 1's
    element before rank 0's (a plausible mistake) changes the entry state."""
    from delta_rule_sequence_b200.workloads import WORKLOADS, make_inputs

    wl = WORKLOADS["tiny"].with_(T=128, s0_std=0.05)
    x = make_inputs(wl, seed=11)
    element, fold, _ = _oracle_steps()
    parts = [{n: (None if t is None or n == "S0" else t[:, a:b].contiguous()) for n, t in x.items()}
             for a, b in ((0, 64), (64, 128))]
    els = [element(p["q"], p["k"], p["v"], p["alpha"], p["beta"], p["u"], p["w"], 64) for p in parts]
    right = fold(fold(x["S0"].double(), *els[0]), *els[1])
    wrong = fold(fold(x["S0"].double(), *els[1]), *els[0])
    import oracle
    _, S_ref = oracle.scan_ref(**x)
    np.testing.assert_allclose(right.numpy(), S_ref, rtol=1e-10, atol=1e-10)
    assert np.abs(wrong.numpy() - S_ref).max() > 1e-3
