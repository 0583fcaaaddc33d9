"""The multi-GPU host path of bench.py on CPU: every rank runs its own replica (the
path needs no exchange between GPUs), the job's time is the slowest rank's (max over
ranks) and the value counts every rank's units. Two gloo ranks stand in for two GPUs;
nothing here touches a GPU."""
import contextlib
import io
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    w = bench.init_ranks("gloo", timeout_s=60)
    ms = bench.max_over_ranks(1.0 + 3.0 * rank, "cpu")       # rank 1 is the slow one
    q.put((rank, w, ms, bench.job_throughput(1000, w, ms)))
    bench.leave_ranks()


def test_two_gloo_ranks_take_the_slowest_time_and_count_every_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g[0] for g in got] == [0, 1]
    for rank, world, ms, value in got:
        assert world == 2
        assert ms == 4.0                                     # max over the ranks
        assert value == pytest.approx(1000 * 2 / 4e-3)       # both ranks' units


def test_one_rank_needs_no_process_group(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    assert bench.init_ranks("gloo") == 1
    assert bench.max_over_ranks(2.5, "cpu") == 2.5
    assert bench.job_throughput(10, 1, 1.0) == pytest.approx(1e4)


def test_reference_arm_prints_on_rank_zero_only():
    sys.path.insert(0, ROOT)
    import bench
    from mamba_selective_scan_sm_b200 import synth
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.run_reference(None, synth.WORKLOADS["tiny"], rank=1)
    assert out.getvalue() == ""
