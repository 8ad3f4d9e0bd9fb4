"""bench.py across ranks, as two gloo processes on CPU (one process per GPU on a GPU node):
the per-rank times reduce to their maximum, the whole-job value counts every rank's work,
and a rank that leaves makes the others fail with an error instead of hanging."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import _multirank_worker as worker  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(target, world, expect, timeout=90):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        return sorted(q.get(timeout=timeout) for _ in range(expect))
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()


def test_times_reduce_to_the_slowest_rank_and_value_counts_all_ranks():
    res = _run(worker.max_worker, 2, 2)
    for rank, times, value in res:
        assert times == [11.0, 23.0]
        assert value == pytest.approx(2 * 5 * 1e12 / 11e-3 / 1e12)


def test_a_rank_that_leaves_is_reported_not_waited_for():
    (rank, outcome, seconds), = _run(worker.dying_worker, 2, 1)
    assert rank == 0
    assert outcome.startswith("error"), outcome
    assert seconds < 60
