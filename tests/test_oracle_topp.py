"""Pins of the oracle's top-p selection (CPU only).

The vAttention pages name top-p as the mass-threshold variant of top-k
selection without a formula. The oracle's reading: the smallest number of the
highest-ranked middle positions whose share of the middle's softmax mass under
the (scaled) ranking scores reaches p. These tests check the selected set
against float64 softmax weights computed here from the caches: it reaches p, it
is minimal, it is a top set, and special values of p reduce to known cases.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.helpers import dense_attention, logical_rows, regions, rel_err_rows, to_f64
from verified_sparse_attention_b200 import synth
from verified_sparse_attention_b200.decoder import params_for

TINY = synth.WORKLOADS["tiny_f32"]
GQA = synth.scaled(synth.WORKLOADS["gqa_32k"], max_ctx=3000, batch=2, num_q_heads=8, num_kv_heads=2)
PAGED = synth.scaled(synth.WORKLOADS["paged_sweep"], max_ctx=3000, min_ctx=900, batch=3,
                     num_q_heads=8, num_kv_heads=2)


def _decode(w, inputs):
    return oracle.decode(oracle.make_problem(w), inputs)


def _middle_weights(inputs, w, b, h):
    """float64 softmax weights (relative to the maximum) of the middle under the group-mean query."""
    n = int(inputs["seq_lens"][b])
    s1, wst, _, _, _ = regions(w, n)
    K = logical_rows(inputs, w, b, h)[s1:wst]
    qbar = to_f64(inputs["q"][b, h * w.group:(h + 1) * w.group]).mean(0)
    r = K @ qbar / math.sqrt(w.head_dim)
    return s1, wst, np.exp(r - r.max())


def _chosen(res, inputs, w, b, h):
    """Middle positions the oracle put in I_f (the top-p part)."""
    n = int(inputs["seq_lens"][b])
    s1, wst, _, _, _ = regions(w, n)
    n_if = int(res["sel_count"][b, h]) - int(res["budgets"][b, h])
    sel = res["sel_idx"][b, h, :n_if]
    return np.array(sorted(j for j in sel if s1 <= j < wst), dtype=np.int64)


@pytest.mark.parametrize("w,num,den", [
    (TINY, 1, 2), (TINY, 9, 10), (TINY, 99, 100),
    (GQA, 1, 2), (GQA, 9, 10), (PAGED, 3, 4),
], ids=lambda v: getattr(v, "name", str(v)))
def test_selected_set_reaches_p_is_minimal_and_is_a_top_set(w, num, den):
    w = w.replace(topp_num=num, topp_den=den)
    inputs = synth.make_inputs(w)
    r = _decode(w, inputs)
    p = num / den
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            s1, wst, wt = _middle_weights(inputs, w, b, h)
            T = _chosen(r, inputs, w, b, h) - s1
            total = wt.sum()
            inside = wt[T]
            outside = np.delete(wt, T)
            assert len(T) >= 1
            # reaches p (fixed-point rounding of the weights: 2^-32 each)
            assert inside.sum() >= p * total * (1 - 1e-6), (b, h, inside.sum() / total)
            # minimal: without its lightest member the set is below p
            assert inside.sum() - inside.min() < p * total * (1 + 1e-6), (b, h)
            # a top set: nothing left out outweighs what was taken (near-ties aside)
            if len(outside):
                assert outside.max() <= inside.min() + 1e-4 * wt.max(), (b, h)


def test_p_one_takes_the_whole_middle_and_is_dense_attention():
    w = GQA.replace(topp_num=1, topp_den=1)
    inputs = synth.make_inputs(w)
    r = _decode(w, inputs)
    for b in range(w.batch):
        n = int(inputs["seq_lens"][b])
        for h in range(w.num_kv_heads):
            assert r["sel_count"][b, h] == n and r["budgets"][b, h] == 0
        for hq in range(w.num_q_heads):
            assert rel_err_rows(r["out"][b, hq], dense_attention(inputs, w, b, hq)) <= 1e-12


def test_tiny_p_takes_only_the_highest_ranked_position():
    w = TINY.replace(topp_num=1, topp_den=1 << 30)
    inputs = synth.make_inputs(w)
    r = _decode(w, inputs)
    for h in range(w.num_kv_heads):
        s1, _, wt = _middle_weights(inputs, w, 0, h)
        T = _chosen(r, inputs, w, 0, h)
        assert len(T) == 1 and T[0] - s1 == int(np.argmax(wt))


def test_one_dominant_key_is_the_whole_top_half():
    # a middle key along the query with a score far above the rest carries more
    # than half of the mass alone, so p = 1/2 takes exactly that key
    w = TINY.replace(topp_num=1, topp_den=2)
    inputs = synth.make_inputs(w)
    j0 = 2000
    for h in range(w.num_kv_heads):
        q = inputs["q"][0, h].clone()
        inputs["k_cache"][0, h, j0] = 40.0 * q / q.norm()
    r = _decode(w, inputs)
    for h in range(w.num_kv_heads):
        assert list(_chosen(r, inputs, w, 0, h)) == [j0]


@pytest.mark.parametrize("n", [4096, 4001])
def test_equal_scores_take_exactly_half_the_middle_lowest_first(n):
    # every key the same: every weight is exactly 1, so p = 1/2 needs exactly
    # ceil(|M| / 2) positions (the cut lands on an exact tie of prefix and target),
    # and equal scores go to the lowest positions
    w = TINY.replace(topp_num=1, topp_den=2)
    inputs = synth.make_inputs(w)
    inputs["k_cache"] = torch.zeros_like(inputs["k_cache"])
    inputs["seq_lens"] = torch.tensor([n], dtype=torch.int32)
    r = _decode(w, inputs)
    s1, wst, mlen, _, _ = regions(w, n)
    for h in range(w.num_kv_heads):
        T = _chosen(r, inputs, w, 0, h)
        assert list(T) == list(range(s1, s1 + (mlen + 1) // 2)), (h, len(T), mlen)


def test_top_p_off_is_the_fixed_k():
    inputs = synth.make_inputs(TINY)
    r0 = _decode(TINY, inputs)
    r1 = _decode(TINY.replace(topp_num=7, topp_den=0), inputs)
    for key in ("sel_idx", "sel_count", "budgets", "head_need"):
        np.testing.assert_array_equal(r0[key], r1[key])


@pytest.mark.parametrize("num,den", [(3, 2), (-1, 2), (1, -2)])
def test_invalid_p_is_rejected(num, den):
    with pytest.raises(ValueError):
        _decode(TINY.replace(topp_num=num, topp_den=den), synth.make_inputs(TINY))


def test_the_binding_passes_p_through():
    w = TINY.replace(topp_num=9, topp_den=10)
    prm = params_for(w, {"num_pages": 1})
    assert (prm.topp_num, prm.topp_den) == (9, 10)
    assert params_for(TINY, {"num_pages": 1}).topp_den == 0
