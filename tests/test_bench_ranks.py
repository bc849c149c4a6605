"""Multi-rank timing logic of bench.py on CPU: two gloo ranks, the job time
is the slowest rank's, and the job rate counts every rank's work."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        elapsed = 100.0 + 50.0 * rank          # rank 1 is slower
        m = bench.max_over_ranks(elapsed, dist)
        rate = bench.job_rate(2.0e9, world, 10, m)
        out.put((rank, m, rate))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_weak_rate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, rate in res:
        assert m == 150.0
        assert rate == pytest.approx(2 * 2.0e9 * 10 / 0.150)


def test_pair_count_matches_brute_force():
    import bench
    for Tq, Tk in [(5, 5), (3, 8), (8, 3), (1, 1), (0, 4), (7, 0), (129, 255)]:
        for causal in (False, True):
            brute = sum(1 for i in range(Tq) for j in range(Tk) if (not causal) or j <= i + Tk - Tq)
            assert bench.pairs_count(Tq, Tk, causal) == brute
        for W in (1, 2, 7, 128, 1000):
            brute = sum(1 for i in range(Tq) for j in range(Tk) if i + Tk - Tq - W < j <= i + Tk - Tq)
            assert bench.pairs_count(Tq, Tk, True, W) == brute


def test_incompatible_modes_are_refused_before_any_device_work(monkeypatch, capsys):
    """Mode combinations bench.py does not run return status 2 from the
    argument checks, which come before anything touches a GPU."""
    import sys
    import bench
    for argv in (["--deterministic", "--fp8", "--workload", "3"], ["--deterministic", "--dropout", "0.1"],
                 ["--deterministic", "--workload", "5"], ["--fp8"], ["--dropout", "1.5"], ["--cp"],
                 ["--window", "0"]):
        monkeypatch.setattr(sys, "argv", ["bench.py"] + argv)
        assert bench.main() == 2, argv
