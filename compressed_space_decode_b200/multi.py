"""Multi-GPU plumbing for the data-parallel decode path.

The (sequence, KV head) units of decode attention are independent, so N GPUs
run N independent shards with no collective on the data path (weak scaling:
each rank keeps the per-GPU workload of one GPU).  The only collectives are
the barrier around the timed region and the max over ranks of the measured
device time.
"""
import os
from dataclasses import replace

import torch
import torch.distributed as dist


def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def shard_workload(wl, rank, world):
    """The workload rank `rank` runs: same shapes, its own seeded data."""
    if world <= 1:
        return wl
    return replace(wl, seed=wl.seed + 7919 * rank, name=f"{wl.name}@rank{rank}")


def max_over_ranks(value, device=None):
    """Max of a float over all ranks (identity without a process group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value, device=None):
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier():
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
