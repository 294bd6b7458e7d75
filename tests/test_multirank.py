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
