"""Host-side arithmetic of bench.py (no GPU): the algorithmic byte counts the roofline divides by,
and the lookup of committed ncu traffic figures by a hash of the kernels' code."""
import os
import re

import bench
from delta_rule_sequence_b200.workloads import WORKLOADS


def test_scan_bytes_of_the_bench_workload_by_hand():
    # B4 H8 T4096, dk = dv = 128, bf16 I/O, GDN write, no S0: per token q, k, v, o at 2 B each
    # plus fp32 alpha and beta; once per head the fp32 exit state.
    tokens = 4 * 8 * 4096
    per_token = 4 * 128 * 2 + 2 * 4
    state = 4 * 8 * 128 * 128 * 4
    assert bench.scan_bytes(WORKLOADS["gdn"]) == tokens * per_token + state == 137363456


def test_scan_bytes_rank_l_counts_every_write_pair_and_the_entry_state():
    wl = WORKLOADS["long"]  # B1 H16 T65536 d128 L2, S0 given
    tokens = 16 * 65536
    per_token = 3 * 128 * 2 + 8 + 2 * (128 + 128) * 2
    state = 16 * 128 * 128 * 4
    assert bench.scan_bytes(wl) == tokens * per_token + 2 * state


def test_decode_bytes_by_hand():
    # per head and step: the fp32 state read and written, q, k, o, alpha, beta, L pairs (u, w)
    per_head = 2 * 128 * 128 * 4 + 3 * 128 * 2 + 8 + 4 * 256 * 2
    assert bench.decode_bytes(WORKLOADS["decode"]) == 256 * 32 * per_head == 1096876032


def test_code_hash_ignores_comments_but_not_code():
    a = "int f(int x) {  // doubles x\n    return 2 * x; /* fast */\n}\n"
    b = "int f(int x) {\n  return 2 * x;\n}  // a different comment\n"
    c = "int f(int x) {\n    return 3 * x;\n}\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)


def test_committed_traffic_is_keyed_by_the_current_code(monkeypatch):
    pat = re.compile(r"bench_traffic:\s*workload=(\S+)\s+kernel=(\S+)\s+source_sha256=(\S+)\s+"
                     r"dram_bytes_per_launch=(\d+)")
    pdir = os.path.join(bench.ROOT, "profiles")
    lines = []
    for name in sorted(os.listdir(pdir)):
        with open(os.path.join(pdir, name)) as f:
            lines += [m.groups() for m in map(pat.search, f) if m]
    assert lines, "the profiles carry bench_traffic lines"
    for workload, kernel, sha, nbytes in lines:
        got = bench.committed_traffic(workload, kernel)
        if sha == bench.kernel_source_hash(kernel):
            assert got == int(nbytes) > 0
    # another code version finds nothing: a figure never outlives the code it was measured on
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kernel: "0" * 16)
    assert all(bench.committed_traffic(w, k) is None for w, k, _, _ in lines)


def test_peaks_come_from_the_measured_file_when_present():
    peaks, kind = bench.load_peaks()
    if os.path.exists(os.path.join(bench.ROOT, "MEASURED_PEAKS.json")):
        assert kind == "measured"
    assert peaks["hbm_gbs"] > 0


def test_cpu_model_is_a_string():
    m = bench.cpu_model()
    assert isinstance(m, str) and m
