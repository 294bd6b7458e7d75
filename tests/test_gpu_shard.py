"""One batch decoded as shards (by KV head or by sequence) through the CUDA path.

The shards run one after another on one GPU, each an ordinary vattn_decode over
its slice with the batch and head offsets of its place in the whole batch; the
concatenated results must match the oracle's single call over the whole batch:
indices, counts, budgets and per-head sizes bit for bit, outputs within the
usual tolerance. (The ranks and the all-gather are tested with gloo on CPU.)
"""
import numpy as np
import pytest
import torch

import oracle
from tests.test_gpu_parity import SMALL, _cuda, _to, compare
from verified_sparse_attention_b200 import ranks, synth
from verified_sparse_attention_b200.decoder import decoder_for, params_for

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode,name,world", [
    ("heads", "gqa", 2), ("heads", "gqa", 4), ("heads", "sparq", 2), ("heads", "loki", 2),
    ("heads", "tiny_f32", 4), ("batch", "paged", 2), ("batch", "paged", 4), ("batch", "gqa", 2),
])
def test_shards_equal_one_call(mode, name, world):
    w = SMALL[name]
    dev = _cuda()
    cpu = synth.make_inputs(w)
    parts = []
    for rank in range(world):
        ws, boff, hoff = ranks.shard_workload(w, mode, world, rank)
        xs = _to(ranks.shard_inputs(cpu, w, mode, world, rank), dev)
        dec = decoder_for(ws)
        try:
            res = dec.decode(xs["q"], xs["k_cache"], xs["v_cache"], xs["page_table"], xs["seq_lens"],
                             params_for(ws, xs, batch_offset=boff, head_offset=hoff))
            torch.cuda.synchronize()
            assert dec.last_error() == 0
            parts.append({k: v.cpu() for k, v in res.items()})
        finally:
            dec.close()
    dim = 0 if mode == "batch" else 1
    got = {k: torch.cat([p[k] for p in parts], dim).numpy() for k in parts[0]}
    ref = oracle.decode(oracle.make_problem(w), cpu)
    compare(w, got, ref, range(w.units))
