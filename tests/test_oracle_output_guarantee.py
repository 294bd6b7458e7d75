"""Pins of the oracle's output (numerator) guarantee, CPU only.

The blog page on vAttention ("How vAttention Works" and the paragraph after
it) says the budget is placed on the softmax denominator as a relaxation of
guaranteeing the attention output. The output guarantee also sizes the sample
so that the numerator vector Nv = sum_j exp(s_j - m) v_j is estimated within
eps (relative, Euclidean length) with probability about 1 - delta. These tests
check that mode against facts outside the oracle: the promised coverage, exact
invariances, and special cases that reduce it to the denominator budget.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.helpers import dense_attention, exact_scores, logical_rows, rel_err_rows
from verified_sparse_attention_b200 import synth

TINY = synth.WORKLOADS["tiny_f32"]
GQA = synth.scaled(synth.WORKLOADS["gqa_32k"], max_ctx=4000, batch=2, num_q_heads=8, num_kv_heads=2)


def _decode(w, inputs, **kw):
    return oracle.decode(oracle.make_problem(w, **kw), inputs)


def _wilson_upper(k, n, zq=2.576):
    ph = k / n
    den = 1 + zq * zq / n
    c = ph + zq * zq / (2 * n)
    a = zq * math.sqrt(ph * (1 - ph) / n + zq * zq / (4 * n * n))
    return (c + a) / den


def _numerator_trials(w, inputs, seeds, guarantee):
    """Per (seed, head): is |Nv_hat - Nv| <= eps |Nv|, with Nv from every position in float64."""
    exact = {}
    for hq in range(w.num_q_heads):
        s = exact_scores(inputs, w, 0, hq)
        V = logical_rows(inputs, w, 0, hq // w.group, "v_cache")
        exact[hq] = (s, V)
    hits, budgets = [], []
    for sd in seeds:
        r = _decode(w, inputs, seed=sd, guarantee=guarantee)
        budgets.append(r["budgets"][0].copy())
        for hq in range(w.num_q_heads):
            s, V = exact[hq]
            nv = (np.exp(s - r["ref_max"][0, hq])[:, None] * V).sum(0)
            nv_hat = r["out"][0, hq] * r["den_hat"][0, hq]
            hits.append(np.linalg.norm(nv_hat - nv) <= float(np.float32(w.eps)) * np.linalg.norm(nv))
    return np.array(hits), np.array(budgets)


def _coherent(inputs):
    """V shifted by +1 per element: the tail's numerator adds up coherently."""
    return dict(inputs, v_cache=inputs["v_cache"] + 1.0)


def test_numerator_coverage_over_500_seeds():
    # eps 0.1 on the tiny config with coherent V keeps the budgets sampled (a few
    # hundred of a 3900-long tail); |Nv_hat - Nv| <= eps |Nv| must hold with
    # probability >= 1 - delta (99% Wilson upper bound)
    w = TINY.replace(eps=0.1)
    inputs = _coherent(synth.make_inputs(w))
    ntail = 4096 - 4 - 64 - 128
    hits, budgets = _numerator_trials(w, inputs, range(500), "output")
    assert (budgets < ntail).all() and (budgets > w.pilot_min).all(), budgets.min()
    assert _wilson_upper(hits.sum(), len(hits)) >= 1 - w.delta, hits.mean()


def test_denominator_budgets_miss_the_numerator_target():
    # the same target with the denominator-only budget misses far more often: the
    # coverage above comes from the numerator's budget term
    w = TINY.replace(eps=0.1)
    inputs = _coherent(synth.make_inputs(w))
    hits, budgets = _numerator_trials(w, inputs, range(200), "denominator")
    assert hits.mean() < 0.85, hits.mean()


@pytest.mark.parametrize("eps", [0.5, 1.0])
def test_incoherent_tail_meets_the_target(eps):
    # zero-mean V: the tail's numerator is noise and the x v terms are heavy-tailed,
    # so a 64-draw pilot overestimates |Nv|^2 several-fold when taken at face value
    # (the unbiased plug-in met the target in about 87 % of trials at eps 0.5). The
    # lower confidence bound takes the whole tail whenever the pilot cannot bound
    # |Nv| away from 0, and the target holds at 1 - delta (99 % Wilson upper bound)
    w = TINY.replace(eps=eps)
    inputs = synth.make_inputs(w)
    hits, _ = _numerator_trials(w, inputs, range(300), "output")
    assert _wilson_upper(hits.sum(), len(hits)) >= 1 - w.delta, hits.mean()


def test_incoherent_tail_is_sampled_when_the_pilot_can_bound_it():
    # a sharper query (q doubled) lets the planted keys carry most of |Nv|, so a
    # 256-draw pilot bounds |Nv| away from 0: zero-mean tails are sampled again,
    # and still meet the target
    w = TINY.replace(eps=0.3, pilot_min=256)
    inputs = synth.make_inputs(w)
    inputs = dict(inputs, q=inputs["q"] * 2.0)
    hits, budgets = _numerator_trials(w, inputs, range(150), "output")
    assert (budgets < 3900).mean() > 0.5, budgets.mean()
    assert _wilson_upper(hits.sum(), len(hits)) >= 1 - w.delta, hits.mean()


@pytest.mark.parametrize("w", [TINY.replace(eps=0.1), GQA.replace(eps=0.3)], ids=lambda w: w.name)
@pytest.mark.parametrize("factor", [2.0, 0.25])
def test_budget_is_invariant_to_power_of_two_scaling_of_v(w, factor):
    # scaling V by a power of two is exact and multiplies tr(Sigma) and |Nv|^2 alike
    inputs = _coherent(synth.make_inputs(w))
    r0 = _decode(w, inputs, guarantee="output")
    scaled = dict(inputs, v_cache=inputs["v_cache"] * factor)
    r1 = _decode(w, scaled, guarantee="output")
    ntail_max = max(int(n) for n in inputs["seq_lens"])
    assert (r0["budgets"] < ntail_max - 300).any()  # some unit is sampled
    np.testing.assert_array_equal(r0["budgets"], r1["budgets"])
    np.testing.assert_array_equal(r0["head_need"], r1["head_need"])
    np.testing.assert_array_equal(r0["sel_idx"], r1["sel_idx"])


@pytest.mark.parametrize("w", [TINY, GQA, GQA.replace(eps=0.2)], ids=lambda w: f"{w.name}-{w.eps}")
def test_constant_v_rows_match_the_denominator_closed_form(w):
    # every V row the same vector c: tr(Sigma) = |c|^2 var(x) and Nv_hat = c D_hat. With
    # a = N_tail^2 var(x) / (p D_hat^2) = n_d eps^2 / (z^2 p) for the denominator's
    # unrounded need n_d, the noise energy is R = |c|^2 D_hat^2 a, the unbiased
    # |Nv|^2 is |c|^2 D_hat^2 (1 - a) and its lower bound
    # L = |c|^2 D_hat^2 ((1 - a) - z sqrt(4 a - 2 a^2)), so
    # n_v = n_d / ((1 - a) - z sqrt(4 a - 2 a^2)), or the whole tail when that is <= 0
    inputs = synth.make_inputs(w)
    g = torch.Generator().manual_seed(7)
    c = torch.randn(w.head_dim, generator=g).to(inputs["v_cache"].dtype)
    const = dict(inputs, v_cache=torch.zeros_like(inputs["v_cache"]) + c)
    rd = _decode(w, const, guarantee="denominator")
    ro = _decode(w, const, guarantee="output")
    z = oracle.z_quantile(w.delta)
    e2 = float(np.float32(w.eps)) ** 2
    checked = whole = 0
    for b in range(w.batch):
        n = int(inputs["seq_lens"][b])
        s1 = min(w.sinks, n)
        wst = max(n - w.window, s1)
        kb = w.topk_abs if w.topk_den == 0 else (n * w.topk_num) // w.topk_den
        ntail = (wst - s1) - min(kb, wst - s1)
        p = w.pilot_min if w.pilot_den == 0 else max(w.pilot_min, -(-n * w.pilot_num // w.pilot_den))
        for hq in range(w.num_q_heads):
            nd = int(rd["head_need"][b, hq])
            nv = int(ro["head_need"][b, hq])
            if nd >= ntail or ntail <= p:
                continue
            def f(x):
                a = x * e2 / (z * z * p)
                den = (1 - a) - z * math.sqrt(max(0.0, 4 * a - 2 * a * a))
                return math.inf if den <= 0 else x / den
            if f(nd) >= ntail:
                assert nv == ntail, (b, hq, nd, nv)
                whole += 1
                continue
            lo, hi = math.ceil(f(nd - 1)) - 1, math.ceil(f(nd)) + 1
            assert lo <= nv <= hi, (b, hq, nd, nv, lo, hi)
            checked += 1
    assert checked >= 4, (checked, whole)


@pytest.mark.parametrize("w", [TINY, GQA], ids=lambda w: w.name)
def test_zero_v_adds_nothing_to_the_budget(w):
    inputs = synth.make_inputs(w)
    zero = dict(inputs, v_cache=torch.zeros_like(inputs["v_cache"]))
    rd = _decode(w, zero, guarantee="denominator")
    ro = _decode(w, zero, guarantee="output")
    for key in ("budgets", "head_need", "sel_idx", "sel_count"):
        np.testing.assert_array_equal(rd[key], ro[key])


def test_output_budget_never_below_the_denominator_budget():
    w = GQA.replace(eps=0.3)
    inputs = _coherent(synth.make_inputs(w))
    rd = _decode(w, inputs, guarantee="denominator")
    ro = _decode(w, inputs, guarantee="output")
    assert (ro["head_need"] >= rd["head_need"]).all()
    assert (ro["budgets"] >= rd["budgets"]).all()
    assert (ro["budgets"] > rd["budgets"]).any()
    # the deterministic set, and the pilot prefix of a sampled tail, do not depend
    # on the guarantee
    sampled = 0
    for b in range(w.batch):
        n = int(inputs["seq_lens"][b])
        for h in range(w.num_kv_heads):
            nI = rd["sel_count"][b, h] - rd["budgets"][b, h]
            assert ro["sel_count"][b, h] - ro["budgets"][b, h] == nI
            ntail = n - nI
            m = nI + (min(rd["budgets"][b, h], ro["budgets"][b, h]) if ro["budgets"][b, h] < ntail else 0)
            sampled += ro["budgets"][b, h] < ntail
            np.testing.assert_array_equal(rd["sel_idx"][b, h, :m], ro["sel_idx"][b, h, :m])
    assert sampled > 0


def test_small_eps_takes_every_tail_and_is_dense_attention():
    w = GQA.replace(eps=0.05)
    inputs = synth.make_inputs(w)
    r = _decode(w, inputs, guarantee="output")
    for b in range(w.batch):
        n = int(inputs["seq_lens"][b])
        for hq in range(w.num_q_heads):
            assert r["sel_count"][b, hq // w.group] == n
            ref = dense_attention(inputs, w, b, hq)
            assert rel_err_rows(r["out"][b, hq], ref) <= 1e-12


def test_unknown_guarantee_is_rejected():
    w = TINY
    pr = oracle.make_problem(w)
    pr.guarantee = 2
    with pytest.raises(ValueError):
        oracle.decode(pr, synth.make_inputs(w))
