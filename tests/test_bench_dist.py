"""bench.py's multi-GPU plumbing on the CPU: two ranks over gloo (127.0.0.1).  Each rank runs
its own replica; the step time is the max over ranks and ``value`` counts every rank's units
(weak scaling).  The reference arm runs on rank 0 only."""
import argparse
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_gloo_time_is_the_max_and_value_counts_both_replicas():
    from tests._dist_worker import worker

    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=worker, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(queue.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, *_ in results] == [0, 1]
    for _, world, ms, value in results:
        assert world == 2
        assert ms == 20.0  # the slower rank's step
        assert value == pytest.approx(4096 * 2 / 0.020)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import bench

    args = argparse.Namespace(gpus=2, steps=1, warmup=0)
    assert bench.run_reference(args, 2, 1) is None
    assert capsys.readouterr().out == ""
