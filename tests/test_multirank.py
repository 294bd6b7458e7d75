"""The multi-GPU host logic (bench.py under torchrun) with two gloo ranks on CPU.

Each rank runs its own batch (weak scaling, no data-path collective); the job's
time is the slowest rank's and its rate counts every rank's calls. Only rank 0
reports.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

from verified_sparse_attention_b200 import ranks, synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        env = ranks.rank_env()
        w = ranks.rank_workload(synth.WORKLOADS["tiny_f32"], rank)
        ms = [12.5, 31.0][rank]  # this rank's elapsed time
        ranks.barrier(world)
        ms_max = ranks.max_over_ranks(ms, world)
        q.put((rank, env, w.data_seed, ms_max, ranks.job_rate(world, 100, ms_max), ranks.reports(rank)))
        ranks.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, env0, seed0, max0, rate0, rep0), (r1, env1, seed1, max1, rate1, rep1) = res
    assert env0 == (2, 0, 0) and env1 == (2, 1, 1)
    assert seed0 != seed1  # own synthetic data per rank, same shapes
    assert max0 == max1 == 31.0  # the slowest rank's time
    assert rate0 == rate1 == pytest.approx(2 * 100 / 0.031)
    assert rep0 and not rep1  # one result line, from rank 0


def test_single_process_defaults(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert ranks.rank_env() == (1, 0, 0)
    w = synth.WORKLOADS["gqa_32k"]
    assert ranks.rank_workload(w, 0) is w
    assert ranks.max_over_ranks(7.0, 1) == 7.0
    assert ranks.job_rate(1, 50, 250.0) == pytest.approx(200.0)


# ------------------------------------------------------------ one batch split over ranks
SHARD_CASES = [
    ("heads", "tiny_f32", dict(max_ctx=2000)),
    ("heads", "gqa_32k", dict(max_ctx=3000, batch=2)),
    ("heads", "loki_64k", dict(max_ctx=2500, batch=2)),
    ("heads", "sparq_128k", dict(max_ctx=2500, batch=2)),
    ("batch", "gqa_32k", dict(max_ctx=3000, batch=4)),
    ("batch", "paged_sweep", dict(max_ctx=3000, min_ctx=1000, batch=4)),
]


def _shard_worker(rank, world, port, q):
    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        results = []
        for mode, name, kw in SHARD_CASES:
            w = synth.scaled(synth.WORKLOADS[name], **kw)
            x = synth.make_inputs(w)                       # the whole batch (same seed on every rank)
            ws, boff, hoff = ranks.shard_workload(w, mode, world, rank)
            xs = ranks.shard_inputs(x, w, mode, world, rank)
            r = oracle.decode(oracle.make_problem(ws, batch_offset=boff, head_offset=hoff), xs)
            mine = {k: torch.from_numpy(np.ascontiguousarray(r[k]))
                    for k in ("out", "sel_idx", "sel_count", "budgets", "head_need")}
            full = ranks.gather_outputs(mine, mode, world)
            if rank == 0:
                ref = oracle.decode(oracle.make_problem(w), x)
                same = {k: bool(np.array_equal(full[k].numpy(), ref[k])) for k in full}
                results.append((mode, name, same, int(ws.units), int(w.units)))
        q.put((rank, results))
        ranks.barrier(world)
    finally:
        dist.destroy_process_group()


def test_one_batch_sharded_over_two_gloo_ranks_equals_one_call():
    # each rank decodes its share of the batch (by KV head or by sequence) with the
    # oracle, the shards are all-gathered, and the result must equal one call over
    # the whole batch bit for bit (outputs included: the same double arithmetic
    # per unit, and the offsets make the shards draw what the whole batch draws)
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert len(res[0]) == len(SHARD_CASES)
    for mode, name, same, shard_units, units in res[0]:
        assert shard_units * world == units
        assert all(same.values()), (mode, name, same)


def test_shards_without_offsets_draw_other_samples():
    # the planted mistake: a shard that numbers its units from 0 draws another
    # sample than the whole batch does for the same units
    import numpy as np

    import oracle
    w = synth.scaled(synth.WORKLOADS["gqa_32k"], max_ctx=3000, batch=2)
    x = synth.make_inputs(w)
    ws, boff, hoff = ranks.shard_workload(w, "heads", 2, 1)
    xs = ranks.shard_inputs(x, w, "heads", 2, 1)
    good = oracle.decode(oracle.make_problem(ws, batch_offset=boff, head_offset=hoff), xs)
    bad = oracle.decode(oracle.make_problem(ws), xs)
    ref = oracle.decode(oracle.make_problem(w), x)
    assert np.array_equal(good["sel_idx"], ref["sel_idx"][:, hoff:])
    assert not np.array_equal(bad["sel_idx"], ref["sel_idx"][:, hoff:])


def test_shard_shapes_and_uneven_splits():
    w = synth.WORKLOADS["gqa_32k"]
    ws, boff, hoff = ranks.shard_workload(w, "heads", 4, 3)
    assert (ws.num_kv_heads, ws.num_q_heads, boff, hoff) == (2, 8, 0, 6)
    ws, boff, hoff = ranks.shard_workload(w, "batch", 8, 5)
    assert (ws.batch, boff, hoff) == (1, 5, 0)
    with pytest.raises(ValueError):
        ranks.shard_workload(w, "heads", 3, 0)
    with pytest.raises(ValueError):
        ranks.shard_workload(w, "rows", 2, 0)
