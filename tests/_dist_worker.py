"""Rank body for the two-process gloo test of bench.py's multi-GPU plumbing (CPU only)."""
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def worker(rank, world, port, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench

    w, r, _ = bench.dist_setup(world, backend="gloo")
    try:
        step_ms = 10.0 * (r + 1)  # the ranks' own step times: 10 ms, 20 ms
        ms = bench.max_over_ranks(step_ms, w)
        bench.barrier(w)
        queue.put((r, w, ms, bench.job_throughput(4096, w, ms)))
    finally:
        torch.distributed.destroy_process_group()
