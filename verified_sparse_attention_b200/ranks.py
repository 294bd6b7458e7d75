"""Host logic of a multi-GPU run (one process per GPU, launched by torchrun).

Two ways to use N GPUs. Replicas (the default of bench.py): each rank runs its
own batch of the same shape on its own GPU (weak scaling), with no data-path
collective; the only collectives are the timing ones (a barrier on both sides
of the timed region and the maximum of the ranks' elapsed times). Sharding:
the ranks split one batch by KV head or by sequence and all-gather the results
(see shard_workload below). Nothing here needs a GPU, so the same functions run
under the gloo backend on CPU.
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


# ------------------------------------------------------------------ sharding one batch
# One decode call's batch split across ranks, either by KV head (each rank holds
# its heads' slice of every cache, as tensor parallelism lays them out) or by
# sequence (each rank holds its sequences). Every unit (sequence, KV head) is
# independent, so a shard is an ordinary decode call over its slice; its draws
# name the units by their place in the whole batch (vattn_params.batch_offset /
# head_offset), so the gathered results equal one call over the whole batch.
SHARD_MODES = ("heads", "batch")


def shard_range(n, world, rank):
    """[first, last) of rank's equal share of n items (n must divide evenly)."""
    if n % world:
        raise ValueError(f"{n} items do not split evenly over {world} ranks")
    per = n // world
    return rank * per, (rank + 1) * per


def shard_workload(w, mode, world, rank):
    """(the shard's workload, batch_offset, head_offset) for rank's share of w."""
    if mode == "heads":
        h0, h1 = shard_range(w.num_kv_heads, world, rank)
        return w.replace(num_kv_heads=h1 - h0, num_q_heads=(h1 - h0) * w.group), 0, h0
    if mode == "batch":
        b0, b1 = shard_range(w.batch, world, rank)
        return w.replace(batch=b1 - b0), b0, 0
    raise ValueError(f"unknown shard mode {mode!r}")


def shard_inputs(x, w, mode, world, rank):
    """Rank's slice of the whole batch's inputs x (the layouts of synth.make_inputs,
    for workload w). By head: q's query heads and every cache's KV heads; by sequence:
    q, lengths and page-table rows, and, for a contiguous cache (one page per
    sequence), its pages with the table renumbered; a paged pool is kept whole."""
    out = dict(x)
    if mode == "heads":
        h0, h1 = shard_range(w.num_kv_heads, world, rank)
        G = w.group
        out["q"] = x["q"][:, h0 * G:h1 * G].contiguous()
        for k in ("k_cache", "v_cache", "k_t_cache", "k_proj_cache"):
            if k in x:
                out[k] = x[k][:, h0:h1].contiguous()
        if "proj_basis" in x:
            out["proj_basis"] = x["proj_basis"][h0:h1].contiguous()
        return out
    b0, b1 = shard_range(w.batch, world, rank)
    out["q"] = x["q"][b0:b1].contiguous()
    out["seq_lens"] = x["seq_lens"][b0:b1].contiguous()
    pt = x["page_table"][b0:b1]
    if w.page_size >= w.max_ctx:  # one page per sequence: page b holds sequence b
        for k in ("k_cache", "v_cache", "k_t_cache", "k_proj_cache"):
            if k in x:
                out[k] = x[k][b0:b1].contiguous()
        pt = torch.where(pt >= 0, pt - b0, pt)
        out["num_pages"] = b1 - b0
    out["page_table"] = pt.contiguous()
    return out


# the output dimension that a shard mode splits: sequence, or (KV or query) head
_SPLIT_DIM = {"batch": 0, "heads": 1}


def gather_outputs(outs, mode, world):
    """The whole batch's outputs from every rank's (all-gather over the process group:
    NCCL on GPUs, gloo on CPU); out, sel_idx, sel_count, budgets and head_need."""
    dim = _SPLIT_DIM[mode]
    full = {}
    for key in sorted(outs):
        t = outs[key].contiguous()
        if world == 1:
            full[key] = t
            continue
        parts = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(parts, t)
        full[key] = torch.cat(parts, dim)
    return full
