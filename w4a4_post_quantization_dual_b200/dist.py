"""Multi-process plumbing for the data-parallel path (one process per GPU).

The DualQuant path shards with no exchange: every m x G column-block tile,
every weight and every token batch is an independent unit, so ranks never
talk on the data path.  The only collectives are host-side bookkeeping:
a barrier around timed regions and the max-over-ranks reduction of the
measured times.  torch.distributed is plumbing here (NCCL on GPUs, gloo on
CPU); nothing in this module computes any part of the method.
"""
import datetime
import os

import torch


def env_ranks():
    """(rank, world, local_rank) from the torchrun environment (defaults: single process)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend, timeout_s=300):
    """Initialise the default process group when more than one rank runs."""
    rank, world, local_rank = env_ranks()
    if world > 1 and not torch.distributed.is_initialized():
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group(backend,
                                             timeout=datetime.timedelta(seconds=timeout_s))
    return rank, world, local_rank


def shard(n_units, rank, world):
    """Round-robin assignment of independent units (weights, tiles) to ranks."""
    return list(range(rank, n_units, world))


def max_over_ranks(values, device=None):
    """Element-wise maximum of a list of floats over all ranks (identity for one rank)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if torch.distributed.is_initialized() and torch.distributed.get_world_size() > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def barrier():
    if torch.distributed.is_initialized() and torch.distributed.get_world_size() > 1:
        torch.distributed.barrier()


def finalize():
    if torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()
