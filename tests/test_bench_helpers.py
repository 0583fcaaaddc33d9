"""CPU checks of the benchmark's bookkeeping: the algorithmic bytes, exp and FP32
operation counts the roofline divides by, and the config it reports, for every
workload (counted by hand here from the shapes)."""
import types

import pytest

import bench
from mamba_selective_scan_sm_b200 import synth

W = synth.WORKLOADS


def test_m130_algorithmic_bytes_and_exps():
    B, D, L, N = 8, 1536, 2048, 16
    act = B * D * L * 2 * 4                       # u, delta, z read, y written (bf16)
    bc = B * N * L * 2 * 2                        # B, C (bf16)
    params = (D * N + 2 * D) * 4 + D * 5 * 4      # A, D, dt bias; conv taps + bias (fp32)
    assert bench.algorithmic_bytes(W["m130"]) == act + bc + params == 202_516_480
    assert bench.exp_count(W["m130"]) == B * D * L * N == 402_653_184


def test_heads_workload_counts():
    w = W["heads128"]
    B, D, L, N = 8, 1536, 2048, 128
    assert bench.exp_count(w) == B * D * L        # one decay exp per (b, d, l) with heads
    assert bench.fp32_ops(w) == 3 * B * D * L * N
    params = (24 + 2 * D) * 4 + D * 5 * 4         # A per head, D, dt bias; conv
    assert bench.algorithmic_bytes(w) == B * D * L * 2 * 4 + B * N * L * 2 * 2 + params


def test_bidirectional_counts_both_directions():
    w = W["bidir"]
    assert bench.exp_count(w) == 2 * 16 * 768 * 1024 * 16
    assert bench.fp32_ops(w) == 2 * 3 * 16 * 768 * 1024 * 16


def test_decode_counts_state_traffic():
    w = W["decode_h128"]
    rows = 256 * 1536
    ab = bench.algorithmic_bytes(w)
    assert ab > rows * 128 * 4 * 2                # the fp32 state read and written dominates
    assert ab < rows * 128 * 4 * 2 * 1.05


@pytest.mark.parametrize("key", sorted(W))
def test_every_workload_has_a_config(key):
    args = types.SimpleNamespace(gpus=1, chunks=0)
    c = bench.config_of(W[key], args)
    assert c["workload"] == W[key].name
    assert "l2" in c
    assert bench.algorithmic_bytes(W[key]) > 0
    if W[key].extra.get("channel_last"):
        assert "layout" in c


def test_passes_per_step_reach_the_minimum_step_time():
    assert bench.passes_for(4.07) == 7                # 7 x 4.07 ms >= 25 ms
    assert bench.passes_for(0.25) == 100
    assert bench.passes_for(30.0) == 1
    assert bench.passes_for(25.0) == 1
    assert bench.passes_for(0.0) == 1
    for ms in (0.03, 0.2517, 2.24, 3.3, 24.9):
        p = bench.passes_for(ms)
        assert p * ms >= bench.STEP_MIN_MS and (p - 1) * ms < bench.STEP_MIN_MS


def test_recorded_traffic_reads_the_json_record(tmp_path):
    digest = bench.kernel_source_digest("scan")
    rec = {"rows": [{"workload": "long", "bytes": 123.0, "sources_sha256": digest},
                    {"workload": "m130", "bytes": 7.0, "sources_sha256": "0" * 64}]}
    p = tmp_path / "traffic.json"
    p.write_text(__import__("json").dumps(rec))
    assert bench.recorded_traffic("long", str(p)) == 123.0
    assert bench.recorded_traffic("m130", str(p)) is None      # taken of other sources
    assert bench.recorded_traffic("bidir", str(p)) is None
    assert bench.recorded_traffic("long", str(tmp_path / "missing.json")) is None


def test_default_workload_is_the_largest_single_gpu_config():
    import sys
    old = sys.argv
    sys.argv = ["bench.py"]
    try:
        assert bench.parse().workload == "long"
    finally:
        sys.argv = old
    w = W["long"]
    assert (w.batch, w.dim, w.seqlen, w.dstate, w.dtype, w.final_state) == (1, 5120, 65536, 16,
                                                                           "bf16", True)


def test_clock_sampler_counts_the_samples_inside_the_timed_window(tmp_path, monkeypatch):
    """A fake nvidia-smi prints one sample every 20 ms; start() returns once the first has
    arrived, and stop() takes the median and the reasons over the window's samples."""
    import os
    import time
    fake = tmp_path / "nvidia-smi"
    fake.write_text("#!/bin/sh\n"
                    "while true; do\n"
                    "  echo '0, 1965, 1965, 300.5, 0x0, Not Active, Not Active, Not Active, Active'\n"
                    "  sleep 0.02\n"
                    "done\n")
    fake.chmod(0o755)
    monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ['PATH']}")
    s = bench.ClockSampler(0)
    s.start()
    assert s.lines, "start() returns after the first sample"
    w0 = time.perf_counter()
    time.sleep(0.3)
    w1 = time.perf_counter()
    time.sleep(0.1)
    c = s.stop((w0, w1))
    assert c["sm_mhz"] == 1965.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]
    assert 5 <= c["samples_under_load"] < c["samples"]
