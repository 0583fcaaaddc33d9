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
