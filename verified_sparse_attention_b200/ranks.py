"""Host logic of a multi-GPU run (one process per GPU, launched by torchrun).

The decode step shards by sequence batch with no data-path collective: each
rank runs its own batch of the same shape on its own GPU (weak scaling). The
only collectives are the timing ones: a barrier on both sides of the timed
region and the maximum of the ranks' elapsed times. Nothing here touches a
GPU, so the same functions run under the gloo backend on CPU.
"""
import os

import torch
import torch.distributed as dist


def rank_env():
    """(world size, rank, local rank) from the torchrun environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_workload(w, rank):
    """The workload rank `rank` runs: the same shapes, its own synthetic data."""
    return w if rank == 0 else w.replace(data_seed=w.data_seed + 1000 * rank)


def barrier(world):
    if world > 1:
        dist.barrier()


def max_over_ranks(value, world, device="cpu"):
    """The largest of the ranks' values (the job's time is its slowest rank's)."""
    if world == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world, calls_per_rank, ms_max):
    """Whole-job calls per second: every rank's calls over the slowest rank's time."""
    return world * calls_per_rank / (ms_max / 1e3)


def reports(rank):
    """Only rank 0 prints the result line (and runs the host-side reference arm)."""
    return rank == 0
