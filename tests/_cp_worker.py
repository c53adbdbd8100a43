"""Rank body for the gloo test of cp_chunk_fwd: real torch.distributed collectives between CPU
processes, the float64 oracle as the compute steps."""
import datetime
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def worker(rank, world, port, queue, mode, g_mu, cuts, seed):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from gated_deltanet_chunked_fwd_b200.cp import cp_chunk_fwd
    from gated_deltanet_chunked_fwd_b200.inputs import make_inputs
    from tests._cp_helpers import oracle_ops, shards

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        x = make_inputs(1, 700, 2, 4, 16, 16, dtype="fp32", seed=seed, s0_std=0.5, g_mu=g_mu)
        sh = shards(x, cuts)[rank]
        try:
            o, ST, taken = cp_chunk_fwd(sh["q"], sh["k"], sh["v"], sh["beta"], sh["g"],
                                        initial_state=x["initial_state"] if rank == 0 else None,
                                        mode=mode, halo_chunks=2, ops=oracle_ops())
            queue.put((rank, o.numpy(), ST.numpy(), taken, None))
        except RuntimeError as e:
            queue.put((rank, None, None, None, str(e)))
    finally:
        dist.destroy_process_group()
