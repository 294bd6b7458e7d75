"""CUDA top-p selection (k_topp, then the count-based select) against the oracle.

The vAttention page names top-k "(or top-p)" selection as the predictor of the
deterministic set. Both sides take the smallest number of the highest-ranked
middle positions whose 2^-32 fixed-point softmax mass reaches p, so selected
indices, counts, budgets and per-head sizes must match bit for bit, outputs
within 2e-3 (bf16) or 1e-5 (fp32) per row, as for the fixed top-k.
"""
import numpy as np
import pytest
import torch

from tests.helpers import regions
from tests.test_gpu_parity import SMALL, W, _cuda, _full_check, _to, check
from verified_sparse_attention_b200 import _abi, synth
from verified_sparse_attention_b200.decoder import decoder_for, params_for

pytestmark = pytest.mark.gpu


def _p(w, num, den):
    return w.replace(topp_num=num, topp_den=den)


def _topk_part(got, w, inputs, b, h):
    n = int(inputs["seq_lens"][b])
    s1, wst, _, _, _ = regions(w, n)
    n_if = int(got["sel_count"][b, h]) - int(got["budgets"][b, h])
    return [j for j in got["sel_idx"][b, h, :n_if] if s1 <= j < wst]


@pytest.mark.parametrize("name,num,den", [
    ("tiny_f32", 1, 2), ("tiny_f32", 9, 10), ("tiny_f32", 99, 100), ("tiny_f32_ragged", 3, 4),
    ("gqa", 1, 2), ("gqa", 9, 10), ("paged", 3, 4), ("sparq", 9, 10), ("loki", 9, 10),
])
def test_parity_reduced(name, num, den):
    check(_p(SMALL[name], num, den))


def test_p_one_takes_the_whole_middle():
    w = _p(SMALL["gqa"], 1, 1)
    got, _ = check(w)
    n = w.max_ctx
    assert (got["sel_count"] == n).all() and (got["budgets"] == 0).all()


def test_p_zero_takes_nothing_from_the_middle():
    w = _p(SMALL["tiny_f32"], 0, 5)
    inputs = synth.make_inputs(w)
    got, _ = check(w, inputs=inputs)
    for h in range(w.num_kv_heads):
        assert _topk_part(got, w, inputs, 0, h) == []


def test_tiny_p_takes_one_position():
    w = _p(SMALL["tiny_f32"], 1, 1 << 30)
    inputs = synth.make_inputs(w)
    got, _ = check(w, inputs=inputs)
    for h in range(w.num_kv_heads):
        assert len(_topk_part(got, w, inputs, 0, h)) == 1


def test_one_dominant_key_is_the_whole_top_half():
    w = _p(SMALL["tiny_f32"], 1, 2)
    inputs = synth.make_inputs(w)
    j0 = 2000
    for h in range(w.num_kv_heads):
        q = inputs["q"][0, h].clone()
        inputs["k_cache"][0, h, j0] = 40.0 * q / q.norm()
    got, _ = check(w, inputs=inputs)
    for h in range(w.num_kv_heads):
        assert _topk_part(got, w, inputs, 0, h) == [j0]


@pytest.mark.parametrize("n", [4096, 4001])
def test_equal_scores_take_half_the_middle_lowest_first(n):
    w = _p(SMALL["tiny_f32"], 1, 2)
    inputs = synth.make_inputs(w)
    inputs["k_cache"] = torch.zeros_like(inputs["k_cache"])
    inputs["seq_lens"] = torch.tensor([n], dtype=torch.int32)
    got, _ = check(w, inputs=inputs)
    s1, _, mlen, _, _ = regions(w, n)
    for h in range(w.num_kv_heads):
        assert _topk_part(got, w, inputs, 0, h) == list(range(s1, s1 + (mlen + 1) // 2))


def test_edge_lengths_paged():
    w = _p(synth.scaled(W["paged_sweep"], max_ctx=3000, min_ctx=3000, batch=8), 9, 10)
    cpu = synth.make_inputs(w)
    cpu["seq_lens"] = torch.tensor([0, 5, 256, 257, 300, 1000, 2999, 3000], dtype=torch.int32)
    check(w, inputs=cpu)


def test_long_context_streamed_select():
    # a middle longer than one CTA's shared memory takes the streamed select after k_topp
    check(_p(synth.scaled(W["gqa_32k"], max_ctx=50000, batch=1, num_q_heads=8, num_kv_heads=2), 4, 5))


def test_full_size_gqa_32k_every_unit():
    _full_check(_p(W["gqa_32k"], 9, 10))


def test_invalid_p_is_rejected():
    w = SMALL["tiny_f32"]
    dev = _cuda()
    x = _to(synth.make_inputs(w), dev)
    dec = decoder_for(w)
    try:
        o = dec.alloc_outputs(w.batch)
        for num, den in ((3, 2), (-1, 2), (1, -2)):
            prm = params_for(w, x)
            prm.topp_num, prm.topp_den = num, den
            rc = _abi.vattn_decode(dec.ctx, x["q"], x["k_cache"], x["v_cache"], x["page_table"],
                                   x["seq_lens"], w.batch, prm, o["out"], o["sel_idx"],
                                   o["sel_count"], o["budgets"], o["head_need"], check=False)
            assert rc == _abi.VATTN_EINVAL, (num, den)
    finally:
        dec.close()
