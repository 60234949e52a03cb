#!/usr/bin/env python
"""Throughput of the chunked gated delta-rule scan forward (tokens/s per layer) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one prism_scan_fwd call over one batch of the headline workload, by default the
long-context one (B=1, H=16, T=65536, dk=dv=128, L=2 projected rank-L write, chunk 128, bf16 I/O,
fp32 state, nonzero S0): the largest of the scan workloads that fit one GPU.  Inputs are device
resident when timing starts; three input batches rotate (each larger than the 126 MB L2), so every
step streams its inputs from HBM.  Steps are replayed from CUDA graphs (one per input batch) so
that host overhead does not leave gaps between kernels.  Timing uses CUDA events on the launching
stream with a barrier and a synchronize on both sides; the reported time is the max over ranks.

With N > 1 (torchrun, one process per GPU) every rank processes its own batch (weak scaling: the
B*H sequences are independent, so there is no collective in the data path).

Besides the headline line's required keys the JSON line carries: roofline (HBM-bound; algorithmic
bytes per call over the summed device time of the call's launches, each launch timed by CUDA
events the library records around it, against the measured copy bandwidth), cpu_baseline (the
fp64 oracle on a bounded sample, rank 0 at N = 1), e2e (through the public API with pinned-host
inputs copied in and the outputs copied back inside the timed region), clocks sampled during the
timed region, and, as secondary measurements: the other two chunked-scan workloads (gdn: B=4,
H=8, T=4096, d=128, Gated-DeltaNet write; recsys: B=32, H=4, T=8192, d=64, L=4), each measured the
same way with its own roofline and oracle baseline; the decode step (B=256, H=32, d=128, L=4); and
the write-term producer on the two rank-L shapes.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# The kernels a step of each bench workload launches, in launch order, and the source files each
# is compiled from (the hash of those files' code keys the committed ncu traffic figures).
STEP_KERNELS = {
    "gdn": ["gdn_prep_kernel", "gdn_state_kernel"],
    "recsys": ["lrank_prep_kernel", "gdn_state_kernel"],
    "long": ["lrank_prep_kernel", "gdn_state_kernel"],
}
_GDN_SOURCES = ["csrc/scan_gdn.cu", "csrc/tc.cuh", "csrc/chunk_common.cuh", "csrc/common.cuh"]
KERNEL_SOURCES = {
    "gdn_prep_kernel": _GDN_SOURCES,
    "lrank_prep_kernel": _GDN_SOURCES,
    "gdn_state_kernel": _GDN_SOURCES,
    "decode_kernel": ["csrc/decode.cu", "csrc/common.cuh"],
    "write_producer_ring_kernel": ["csrc/producer.cu", "csrc/producer.cuh", "csrc/chunk_common.cuh",
                              "csrc/tc.cuh", "csrc/common.cuh"],
}


def _code_only(text):
    """C++ source without its comments and with runs of blank space folded, so that editing a
    comment does not invalidate a traffic figure measured on the same code."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash(kernel):
    pkg = os.path.join(ROOT, "delta_rule_sequence_b200")
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.normpath(os.path.join(pkg, rel)), encoding="utf-8") as f:
            h.update(os.path.basename(rel).encode() + b"\0" + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def committed_traffic(workload, kernel):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on this source."""
    if kernel not in KERNEL_SOURCES:
        return None
    src = kernel_source_hash(kernel)
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    pat = re.compile(r"bench_traffic:\s*workload=(\S+)\s+kernel=(\S+)\s+source_sha256=(\S+)\s+"
                     r"dram_bytes_per_launch=(\d+)")
    for name in sorted(os.listdir(pdir)):
        if not name.endswith((".md", ".txt")):
            continue
        with open(os.path.join(pdir, name)) as f:
            for line in f:
                m = pat.search(line)
                if m and m.group(1) == workload and m.group(2) == kernel and m.group(3) == src:
                    return int(m.group(4))
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid):
        self.gpu = gpu_uuid
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [c.strip() for c in line.split(",")]))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self.thread:
                self.thread.join(timeout=2)

    def summary(self, t0, t1):
        rows = [r for t, r in self.rows if t0 - 0.15 <= t <= t1 + 0.15] or [r for _, r in self.rows]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        smax = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for n, v in zip(names, r[4:8]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        power = [float(r[2]) for r in rows if re.match(r"^[\d.]+$", r[2])]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max(power) if power else None}


# ------------------------------------------------------------------------------------------------
# algorithmic work of one scan-forward call (what must cross HBM / be computed at minimum)

def scan_bytes(wl, io_bytes=2, with_S0=None):
    B, T, H, dk, dv, L = wl.B, wl.T, wl.H, wl.dk, wl.dv, wl.L
    tok = B * T * H
    per_tok = (2 * dk + dv) * io_bytes + 8  # q, k, o + alpha, beta
    if wl.write == "gdn":
        per_tok += dv * io_bytes
    else:
        per_tok += L * (dk + dv) * io_bytes
    state = B * H * dv * dk * 4
    s0 = state if (with_S0 if with_S0 is not None else wl.s0_std > 0) else 0
    return tok * per_tok + state + s0


def scan_flops(wl):
    """Algorithmic FLOPs of the chunked form (triangular products at half)."""
    C, d, L = wl.chunk, wl.dk, wl.L
    if wl.write == "gdn":
        per = 5 * C * d + C * C / 3 + 6 * d * d
    else:
        per = C * d * (5 + 4 * L) + C * C / 3 + d * d * (6 + 2 * L)
    return wl.B * wl.T * wl.H * per


def producer_bytes(wl):
    """Algorithmic bytes of one write-producer call: per token x, v in and the L pairs (u, w) out
    at bf16, beta in fp32; per head the weights [W_k; W_p] (bf16) and the ShortConv taps (fp32)."""
    d, L = wl.dk, wl.L
    tok = wl.B * wl.T * wl.H
    return tok * (2 * d * 2 + 4 * L + 2 * L * d * 2) + wl.H * (L * 2 * d * d * 2 + 4 * d * 4)


def producer_flops(wl):
    """The 2L projections of every token's anchor (W_k a, W_p a: 2 FLOPs a multiply-add)."""
    return wl.B * wl.T * wl.H * 2 * (2 * wl.L * wl.dk * wl.dk)


def decode_bytes(wl, io_bytes=2):
    heads = wl.B * wl.H
    per = 2 * wl.dv * wl.dk * 4 + (2 * wl.dk + wl.dv) * io_bytes + 8
    per += wl.L * (wl.dk + wl.dv) * io_bytes
    return heads * per


# ------------------------------------------------------------------------------------------------

def cpu_model():
    """The host CPU's model name (from /proc/cpuinfo), or "unknown"."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


ORACLE_WINDOW = 4096  # tokens of each sequence the oracle baselines run over (throughput of the
                      # token recurrence does not depend on where in the sequence a window sits)


def cpu_oracle_sample(wl, budget_s=12.0, n_threads=None):
    """Time the fp64 oracle on (b, h) sequences of the workload, each over its first
    min(T, ORACLE_WINDOW) tokens.  Returns (tokens/s, description, threads).  One sequence is
    timed alone first to size a sample of about `budget_s` seconds on all threads."""
    import oracle
    from delta_rule_sequence_b200.workloads import make_inputs, select_heads

    threads = n_threads or oracle.default_threads()
    Ts = min(wl.T, ORACLE_WINDOW)
    x = make_inputs(wl.with_(T=Ts), seed=0)
    heads_all = [(b, h) for b in range(wl.B) for h in range(wl.H)]
    sub = select_heads(x, heads_all[:1])
    t0 = time.perf_counter()
    oracle.scan_ref(**sub, n_threads=1)
    t1 = time.perf_counter() - t0
    n = max(1, min(len(heads_all), int(budget_s * threads / max(t1, 1e-3))))
    n = max(1, (n // threads) * threads) if n >= threads else n
    sub = select_heads(x, heads_all[:n])
    passes = 0
    t0 = time.perf_counter()
    while True:  # whole passes over the sample until the time budget is used
        oracle.scan_ref(**sub, n_threads=threads)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s or passes >= 1000:
            break
    tokens = passes * n * Ts / wl.H  # a token carries all H heads
    desc = (f"{passes} pass(es) over {n} of {wl.B * wl.H} (b,h) sequences of the {wl.name} "
            f"workload, first {Ts} of T={wl.T} tokens each, fp64 token recurrence on {threads} "
            f"threads, {dt:.1f} s; tokens/s = passes*sequences*tokens/H/s")
    return tokens / dt, desc, threads


def run_reference(args, rank):
    """The base contract's reference arm: the fp64 oracle on the host cores, per step a bounded
    sample of the same workload (one (b,h) sequence per thread, over its first
    min(T, ORACLE_WINDOW) tokens)."""
    if rank != 0:
        return
    import oracle
    from delta_rule_sequence_b200.workloads import WORKLOADS, make_inputs, select_heads

    wl = WORKLOADS[args.workload]
    threads = oracle.default_threads()
    Ts = min(wl.T, ORACLE_WINDOW)
    x = make_inputs(wl.with_(T=Ts), seed=0)
    heads_all = [(b, h) for b in range(wl.B) for h in range(wl.H)]
    per_step = min(len(heads_all), threads)
    subs = [select_heads(x, [heads_all[(s * per_step + i) % len(heads_all)]
                             for i in range(per_step)]) for s in range(2)]
    for i in range(args.warmup):
        oracle.scan_ref(**subs[i % 2], n_threads=threads)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle.scan_ref(**subs[i % 2], n_threads=threads)
    dt = time.perf_counter() - t0
    tokens = args.steps * per_step * Ts / wl.H
    value = tokens / dt
    desc = (f"per step {per_step} (b,h) sequences of the {wl.name} workload, first {Ts} of "
            f"T={wl.T} tokens each, fp64 oracle on {threads} threads")
    line = {
        "impl": "reference", "metric": "scan-fwd tokens/s per layer", "value": value,
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": desc, "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


class ScanBench:
    """One chunked-scan workload on one rank: three seeded input batches resident on the device
    (rotated, so that steps stream their inputs from HBM rather than L2), one CUDA graph per batch
    for the throughput, and the library's per-launch events for the kernel durations."""

    def __init__(self, wl, dev, stream, rank):
        import torch

        from delta_rule_sequence_b200 import prism
        from delta_rule_sequence_b200.workloads import make_inputs

        self.wl, self.dev, self.stream = wl, dev, stream
        self.host_sets = [make_inputs(wl, seed=3 * rank + i) for i in range(3)]
        self.sets = [{n: (None if t is None else t.to(dev)) for n, t in s.items()}
                     for s in self.host_sets]
        self.o = [torch.empty((wl.B, wl.T, wl.H, wl.dv), dtype=wl.torch_io, device=dev)
                  for _ in range(3)]
        self.S = [torch.empty((wl.B, wl.H, wl.dv, wl.dk), dtype=torch.float32, device=dev)
                  for _ in range(3)]
        self.shape = prism.make_shape(self.sets[0]["q"], self.sets[0]["v"], self.sets[0]["u"],
                                      wl.chunk)
        self.ws = prism.workspace_for(self.shape, dev)
        self.launches = prism.prism_scan_fwd_launch_count(self.shape)
        self.graphs = []

    def step(self, i, workspace=None, o=None, S=None, x=None):
        from delta_rule_sequence_b200 import prism

        x = x if x is not None else self.sets[i % 3]
        prism.prism_scan_fwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["u"], x["w"],
                             x["S0"], chunk=self.wl.chunk, o=o if o is not None else self.o[i % 3],
                             S_final=S if S is not None else self.S[i % 3],
                             workspace=workspace if workspace is not None else self.ws,
                             stream=self.stream)

    def capture(self):
        import torch

        with torch.cuda.stream(self.stream):
            for i in range(3):
                self.step(i)
        self.stream.synchronize()
        for i in range(3):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                self.step(i)
            self.graphs.append(g)
        torch.cuda.synchronize()

    def check_status(self, where):
        from delta_rule_sequence_b200 import prism

        status = prism.prism_query_device_status(self.ws, self.stream)
        if status != prism.PRISM_OK:
            raise SystemExit(f"bench: device status {where} ({self.wl.name}): "
                             f"{prism.status_string(status)}")

    def run_graphs(self, n, start=0):
        import torch

        with torch.cuda.stream(self.stream):
            for i in range(start, start + n):
                self.graphs[i % 3].replay()

    def timed_graphs(self, steps, barrier, max_over_ranks):
        """Device time of `steps` graph-replayed steps: ms in total (max over ranks)."""
        import torch

        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(self.stream):
            e0.record(self.stream)
            for i in range(steps):
                self.graphs[i % 3].replay()
            e1.record(self.stream)
        torch.cuda.synchronize()
        barrier()
        return max_over_ranks(e0.elapsed_time(e1))

    def launch_times(self, steps, barrier, max_over_ranks):
        """Average device time of each launch of a step (CUDA events the library records on the
        launching stream around each launch), over `steps` steps launched without graphs.
        Returns (ms per launch, ms per step of that region)."""
        import torch

        from delta_rule_sequence_b200 import prism

        n = self.launches
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(steps)]
        with torch.cuda.stream(self.stream):
            for row in evs:  # record once so that every event handle exists
                for e in row:
                    e.record(self.stream)
        torch.cuda.synchronize()
        barrier()
        p0 = torch.cuda.Event(enable_timing=True)
        p1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.stream):
            p0.record(self.stream)
            for i in range(steps):
                prism.record_launch_events(evs[i])
                self.step(i)
            p1.record(self.stream)
        torch.cuda.synchronize()
        barrier()
        per_step = max_over_ranks(p0.elapsed_time(p1)) / steps
        launch_ms = [max_over_ranks(sum(r[j].elapsed_time(r[j + 1]) for r in evs) / steps)
                     for j in range(n)]
        return launch_ms, per_step

    def release(self):
        for g in self.graphs:
            g.reset()
        self.graphs = []


def scan_roofline(wl, launch_ms, peaks, peaks_kind, timing):
    """Roofline of one scan call.  The algorithmic bytes are defined for the whole path (inputs read
    once, outputs and the state written once), which the call's launches share, so the unit is the
    call: algorithmic bytes per call over the summed device time of its launches."""
    names = STEP_KERNELS.get(wl.name, [])
    if len(names) != len(launch_ms):
        names = [f"launch{j}" for j in range(len(launch_ms))]
    kernels = [{"name": n, "ms_per_launch": launch_ms[j],
                "share": launch_ms[j] / max(1e-12, sum(launch_ms)),
                "dram_bytes_per_launch": committed_traffic(wl.name, n)}
               for j, n in enumerate(names)]
    dominant = max(range(len(launch_ms)), key=lambda j: launch_ms[j])
    alg = scan_bytes(wl)
    kern_ms = sum(launch_ms)
    achieved = alg / (kern_ms / 1e3) / 1e9
    traffic = [k["dram_bytes_per_launch"] for k in kernels]
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"],
            "traffic": sum(traffic) if all(t is not None for t in traffic) else None,
            "peak_kind": f"{peaks_kind} copy bandwidth (burst)",
            "unit_of_work": "one call: " + " + ".join(names),
            "dominant_kernel": names[dominant], "kernels": kernels,
            "algorithmic_bytes_per_step": alg, "algorithmic_flops_per_step": scan_flops(wl),
            "tensor_frac_algorithmic": scan_flops(wl) / (kern_ms / 1e3) / 1e12 / peaks["bf16_tflops"],
            "timing": timing}


def secondary_scan(wl, dev, stream, peaks, peaks_kind, rank, max_over_ranks, barrier, world,
                   steps, warmup, cpu_budget):
    """A scan workload measured like the headline (rotated inputs, graph-replayed steps, per-launch
    events), with its own roofline and, on rank 0 at N = 1, its own oracle baseline."""
    sb = ScanBench(wl, dev, stream, rank)
    sb.capture()
    sb.run_graphs(warmup)
    stream.synchronize()
    sb.check_status("after warm-up")
    ms = sb.timed_graphs(steps, barrier, max_over_ranks) / steps
    launch_ms, probe_ms = sb.launch_times(steps, barrier, max_over_ranks)
    sb.check_status("after timing")
    sb.release()
    out = {"workload": workload_config(wl)["workload"], "ms_per_call": ms,
           "tokens_per_s": world * wl.B * wl.T / (ms / 1e3), "launches": sb.launches,
           "steps": steps, "warmup": warmup,
           "roofline": scan_roofline(wl, launch_ms, peaks, peaks_kind,
                                     f"CUDA events recorded by the library around each launch, "
                                     f"{steps} calls without graphs ({probe_ms:.4f} ms/call there)"),
           "cpu_baseline": None}
    del sb
    if rank == 0 and world == 1 and cpu_budget > 0:
        v, desc, threads = cpu_oracle_sample(wl, budget_s=cpu_budget)
        out["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                               "sample": desc, "cpu_model": cpu_model()}
    return out


def time_producer(wl, dev, stream, peaks, rank, max_over_ranks, barrier, world, steps=20):
    """The write-term producer on a scan workload's shape (random weights), timed alone."""
    import torch

    from delta_rule_sequence_b200 import prism
    from delta_rule_sequence_b200.workloads import make_producer_inputs

    p = {n: t.to(dev) for n, t in make_producer_inputs(wl, seed=7 + rank).items()}
    u = torch.empty((wl.B, wl.T, wl.H, wl.L, wl.dk), dtype=torch.bfloat16, device=dev)
    w = torch.empty_like(u)

    def call():
        prism.prism_write_producer(p["x"], p["v"], p["conv"], p["Wk"], p["Wp"], p["beta"], u=u, w=w,
                                   stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(3):
            call()
    stream.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    with torch.cuda.stream(stream):
        for row in evs:
            for e in row:
                e.record(stream)
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(steps):
            prism.record_launch_events(evs[i])
            call()
        e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    status = prism.prism_query_device_status(None, stream)
    if status != prism.PRISM_OK:
        raise SystemExit(f"bench: device status after the producer: {prism.status_string(status)}")
    ms = max_over_ranks(e0.elapsed_time(e1)) / steps
    kern_ms = sum(r[0].elapsed_time(r[1]) for r in evs) / steps
    alg, fl = producer_bytes(wl), producer_flops(wl)
    achieved = alg / (kern_ms / 1e3) / 1e9
    del p, u, w
    return {"workload": f"write producer on {wl.name}: B={wl.B} H={wl.H} T={wl.T} d={wl.dk} L={wl.L} "
                        f"bf16 I/O, random weights",
            "ms_per_call": ms, "tokens_per_s": world * wl.B * wl.T / (ms / 1e3), "launches": 1,
            "ms_per_launch": {"write_producer_ring_kernel": kern_ms},
            "dram_bytes_per_launch": {"write_producer_ring_kernel":
                                      committed_traffic("producer_" + wl.name, "write_producer_ring_kernel")},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "algorithmic_bytes": alg, "algorithmic_flops": fl,
                         "tensor_frac_algorithmic": fl / (kern_ms / 1e3) / 1e12 / peaks["bf16_tflops"]},
            "steps": steps}


FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # 148 SMs x 128 fp32 FMA lanes x 2 x 1965 MHz


def backward_bytes(wl, io_bytes=2):
    """Algorithmic bytes of one backward call: the forward's inputs and dO read once, every
    gradient written once in fp32, S0 and dS_final read and dS0 written."""
    B, T, H, dk, dv, L = wl.B, wl.T, wl.H, wl.dk, wl.dv, wl.L
    tok = B * T * H
    rd = (2 * dk + dv) * io_bytes + 8                     # q, k, dO, alpha, beta
    wr = (2 * dk) * 4 + 8                                 # dq, dk, dalpha, dbeta
    if wl.write == "gdn":
        rd += dv * io_bytes
        wr += dv * 4
    else:
        rd += L * (dk + dv) * io_bytes
        wr += L * (dk + dv) * 4
    return tok * (rd + wr) + 3 * B * H * dv * dk * 4


def backward_flops(wl):
    """FLOPs of the reverse recurrence itself (one forward step and one backward step per token
    and value row; the kernel's recomputation of the forward is not counted)."""
    L = 1 if wl.write == "gdn" else wl.L
    return wl.B * wl.T * wl.H * wl.dv * wl.dk * (18 + 5 * L)


def time_backward(wl, dev, stream, peaks, rank, max_over_ranks, barrier, world, steps=5):
    """prism_scan_bwd on a scan workload, timed alone (device-resident inputs and dO)."""
    import torch

    from delta_rule_sequence_b200 import prism
    from delta_rule_sequence_b200.workloads import make_inputs

    x = {n: (None if t is None else t.to(dev)) for n, t in make_inputs(wl, seed=7 + rank).items()}
    g = torch.Generator().manual_seed(11 + rank)
    dO = torch.randn((wl.B, wl.T, wl.H, wl.dv), generator=g).to(wl.torch_io).to(dev)
    dS = (torch.randn((wl.B, wl.H, wl.dv, wl.dk), generator=g) * 0.1).float().to(dev)

    def call():
        return prism.prism_scan_bwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["u"], x["w"],
                                    x["S0"], dO=dO, dS_final=dS, stream=stream)

    with torch.cuda.stream(stream):
        call()
    stream.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(steps):
            call()
        e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1)) / steps
    alg, fl = backward_bytes(wl), backward_flops(wl)
    del x, dO, dS
    return {"workload": f"backward on {workload_config(wl)['workload']}",
            "ms_per_call": ms, "tokens_per_s": world * wl.B * wl.T / (ms / 1e3), "launches": 1,
            "roofline": {"bound": "alu", "achieved": fl / (ms / 1e3) / 1e12,
                         "peak": FP32_ALU_TFLOPS, "unit": "TFLOP/s",
                         "frac": fl / (ms / 1e3) / 1e12 / FP32_ALU_TFLOPS,
                         "peak_kind": "fp32 CUDA-core FMA peak from unit counts and the 1965 MHz clock",
                         "algorithmic_flops": fl, "algorithmic_bytes": alg,
                         "hbm_frac": alg / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]},
            "steps": steps,
            "timing": "CUDA events around the calls (each call clears the summed gradients first)"}


def workload_config(wl):
    return {"workload": f"{wl.name}: B={wl.B} H={wl.H} T={wl.T} dk={wl.dk} dv={wl.dv} L={wl.L} "
                        f"chunk={wl.chunk} io={wl.io} state=f32 write={wl.write}",
            "global_batch": wl.B, "seq_len": wl.T, "heads": wl.H,
            "l2": "3 rotating input batches (each > L2 / 3) so inputs stream from HBM"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long")
    ap.add_argument("--decode-steps", type=int, default=200)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the secondary scan workloads and the write producer")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="override the headline workload's T (small cases for profiler captures)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank)
        return

    import torch
    import torch.distributed as dist

    from delta_rule_sequence_b200 import prism
    from delta_rule_sequence_b200.workloads import WORKLOADS, make_decode_state, make_decode_step

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        if world == 1:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    peaks, peaks_kind = load_peaks()
    wl = WORKLOADS[args.workload]
    if args.seq_len > 0:
        wl = wl.with_(T=args.seq_len)
    stream = torch.cuda.Stream(device=dev)

    # ---- the headline workload: three seeded batches per rank, device resident, one CUDA graph
    # per batch, steps rotating over them
    sb = ScanBench(wl, dev, stream, rank)
    sb_launches = sb.launches
    sb.capture()
    sb.run_graphs(args.warmup)
    stream.synchronize()
    sb.check_status("after warm-up")

    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    sampler.start()
    time.sleep(0.3)
    wall0 = time.time()
    ms_total = sb.timed_graphs(args.steps, barrier, max_over_ranks)
    wall1 = time.time()
    sampler.stop()
    ms_per_step = ms_total / args.steps
    tokens_per_step = wl.B * wl.T
    value = world * tokens_per_step * args.steps / (ms_total / 1e3)
    sb.check_status("after timing")
    clocks = sampler.summary(wall0, wall1)

    # ---- per-kernel durations: a second timed region of the same steps, launched without graphs,
    # with the library recording CUDA events on the launching stream around every launch
    launch_ms, probe_ms = sb.launch_times(args.steps, barrier, max_over_ranks)
    roofline = scan_roofline(wl, launch_ms, peaks, peaks_kind,
                             f"CUDA events recorded by the library on the launching stream around "
                             f"each launch, {args.steps} steps without graphs "
                             f"({probe_ms:.4f} ms/step there)")
    sb.release()

    # ---- end to end through the public API: pinned host inputs in, outputs back, every step.
    # Copies in, scans and copies out run on three streams with two device buffers each (a caller
    # streaming batches would do the same): step i's host-to-device copy overlaps step i-1's scan
    # and step i-2's copy back; every step still moves its own inputs and results.
    e2e = None
    if args.e2e_steps > 0:
        pinned = {n: (None if t is None else t.pin_memory()) for n, t in sb.host_sets[0].items()}
        o_host = torch.empty(sb.o[0].shape, dtype=sb.o[0].dtype).pin_memory()
        S_host = torch.empty(sb.S[0].shape, dtype=torch.float32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in pinned.values() if t is not None)
        d2h = o_host.numel() * o_host.element_size() + S_host.numel() * 4
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        dbuf = [sb.sets[0], sb.sets[1]]
        ws2 = [sb.ws, torch.zeros_like(sb.ws)]
        n_e2e = args.e2e_steps

        def run_e2e(nsteps):
            ev_in = [torch.cuda.Event() for _ in range(nsteps)]
            ev_cmp = [torch.cuda.Event() for _ in range(nsteps)]
            ev_out = [torch.cuda.Event() for _ in range(nsteps)]
            for i in range(nsteps):
                x, bi = dbuf[i % 2], i % 2
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_cmp[i - 2])  # the scan that read this buffer is done
                    for n, t in pinned.items():
                        if t is not None:
                            x[n].copy_(t, non_blocking=True)
                    ev_in[i].record(s_in)
                with torch.cuda.stream(stream):
                    stream.wait_event(ev_in[i])
                    if i >= 2:
                        stream.wait_event(ev_out[i - 2])  # the copy back of this output is done
                    sb.step(bi, workspace=ws2[bi], o=sb.o[bi], S=sb.S[bi], x=x)
                    ev_cmp[i].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_cmp[i])
                    o_host.copy_(sb.o[bi], non_blocking=True)
                    S_host.copy_(sb.S[bi], non_blocking=True)
                    ev_out[i].record(s_out)
            return ev_out[-1]

        run_e2e(3)
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        stream.wait_event(e0)
        s_out.wait_event(e0)
        last = run_e2e(n_e2e)
        s_out.wait_event(last)
        e1.record(s_out)
        torch.cuda.synchronize()
        barrier()
        ems = max_over_ranks(e0.elapsed_time(e1))
        sb.check_status("after the end-to-end run")
        e2e = {"value": world * tokens_per_step * n_e2e / (ems / 1e3),
               "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "steps": n_e2e, "ms_per_step": ems / n_e2e,
               "schedule": "copy in / scan / copy out on three streams, two buffers each"}
        del pinned, o_host, S_host, ws2, dbuf
    del sb

    # ---- secondary: the other chunked-scan workloads, measured the same way
    others = {}
    if not args.no_configs:
        for name in ("gdn", "recsys", "long"):
            if name == args.workload:
                continue
            others[name] = secondary_scan(
                WORKLOADS[name], dev, stream, peaks, peaks_kind, rank, max_over_ranks, barrier,
                world, steps=max(20, min(args.steps, 200)), warmup=args.warmup,
                cpu_budget=0.0 if args.no_cpu_baseline else 6.0)

    # ---- secondary: the decode step (B=256, H=32, d=128, L=4), state in HBM, in place
    decode = None
    if args.decode_steps > 0:
        dwl = WORKLOADS["decode"]
        st = make_decode_state(dwl, seed=rank)
        S = st["S0"].to(dev)
        pool = [{n: (None if t is None else t.to(dev)) for n, t in
                 make_decode_step(dwl, st, s, seed=rank).items()} for s in range(4)]
        o_d = torch.empty((dwl.B, 1, dwl.H, dwl.dv), dtype=torch.bfloat16, device=dev)

        def dstep(i):
            x = pool[i % 4]
            prism.prism_step_decode(x["q"], x["k"], None, x["alpha"], x["beta"], x["u"], x["w"],
                                    S, o=o_d, stream=stream)
        with torch.cuda.stream(stream):
            for i in range(10):
                dstep(i)
        torch.cuda.synchronize()
        barrier()
        d0 = torch.cuda.Event(enable_timing=True)
        d1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            d0.record(stream)
            for i in range(args.decode_steps):
                dstep(i)
            d1.record(stream)
        torch.cuda.synchronize()
        barrier()
        if prism.prism_query_device_status(None, stream) != prism.PRISM_OK:
            raise SystemExit("bench: device status after the decode steps")
        dms = max_over_ranks(d0.elapsed_time(d1)) / args.decode_steps
        db = decode_bytes(dwl)
        decode = {"workload": "decode: B=256 H=32 dk=dv=128 L=4 bf16 I/O, fp32 state in place",
                  "ms_per_step": dms, "tokens_per_s": world * dwl.B / (dms / 1e3),
                  "achieved_gbs": db / (dms / 1e3) / 1e9,
                  "frac_of_measured_copy": db / (dms / 1e3) / 1e9 / peaks["hbm_gbs"],
                  "frac_of_8tbs": db / (dms / 1e3) / 1e9 / 8000.0,
                  "bytes_per_step": db, "steps": args.decode_steps,
                  "inputs": "4 seeded step batches cycled; state carried across steps"}
        del S, pool, o_d

    # ---- secondary: the write-term producer on the two rank-L shapes, and the backward pass
    if not args.no_configs:
        for name in ("recsys", "long"):
            others["producer_" + name] = time_producer(WORKLOADS[name], dev, stream, peaks, rank,
                                                       max_over_ranks, barrier, world)
        for name, steps in (("gdn", 5), ("long", 2)):
            others["backward_" + name] = time_backward(WORKLOADS[name], dev, stream, peaks, rank,
                                                       max_over_ranks, barrier, world, steps=steps)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc, threads = cpu_oracle_sample(wl)
        cpu = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": desc,
               "cpu_model": cpu_model()}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": "scan-fwd tokens/s per layer", "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(wl), parallelism=f"dp{world} over (b,h) sequences"),
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": sb_launches * args.steps, "clocks": clocks, "decode": decode,
        "other_workloads": others or None,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
