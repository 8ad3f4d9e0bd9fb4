"""Rank processes for the multi-rank tests (gloo on CPU) of bench.py's cross-rank logic:
every rank times the same work and the job is as slow as its slowest rank."""
import datetime
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _init(rank, world, port, timeout_s):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s))
    return dist


def max_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch

    import bench
    dist = _init(rank, world, port, 30)
    try:
        times = bench.max_over_ranks([10.0 + rank, 20.0 + 3 * rank], dist, torch.device("cpu"))
        q.put((rank, times, bench.whole_job_tflops(world, 5, 1e12, times[0])))
    finally:
        dist.destroy_process_group()


def dying_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch

    import bench
    dist = _init(rank, world, port, 10)
    if rank == 1:
        os._exit(3)   # this rank leaves between steps, with no collective in flight
    t0 = time.time()
    try:
        bench.max_over_ranks([1.0], dist, torch.device("cpu"))
        q.put((rank, "no error", time.time() - t0))
    except Exception as e:   # the survivor learns of it from the collective, not by hanging
        q.put((rank, "error: " + type(e).__name__, time.time() - t0))
