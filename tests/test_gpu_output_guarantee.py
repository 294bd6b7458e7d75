"""CUDA path with the output (numerator) guarantee against the oracle.

Same bar as the denominator-only parity tests: selected indices, counts,
budgets and per-head sizes bit for bit (the numerator sizes are computed in
double in a fixed order on both sides), outputs within 2e-3 (bf16) or 1e-5
(fp32) per row. Coherent V (every element shifted by +1) keeps most budgets
sampled; zero-mean V mostly takes every tail whole, since a small pilot cannot
bound |Nv| away from 0 there.
"""
import numpy as np
import pytest
import torch

from tests.test_gpu_parity import SMALL, W, _cuda, _full_check, check
from verified_sparse_attention_b200 import _abi, synth
from verified_sparse_attention_b200.decoder import decoder_for, params_for

pytestmark = pytest.mark.gpu


def _out(w, **kw):
    return w.replace(guarantee="output", **kw)


def _coherent(w):
    x = synth.make_inputs(w)
    x["v_cache"] = x["v_cache"] + 1.0
    return x


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("eps", [0.1, 0.3])
def test_parity_reduced_coherent_v(name, eps):
    w = _out(SMALL[name], eps=eps)
    got, _ = check(w, inputs=_coherent(w))
    assert (got["budgets"] > 0).any()


@pytest.mark.parametrize("name", ["tiny_f32", "gqa", "paged"])
def test_parity_reduced_zero_mean_v(name):
    check(_out(SMALL[name], eps=0.5))


def test_parity_sampled_numerator_budgets():
    # the sampled branch of the lower confidence bound: a sharper query lets the
    # planted keys carry |Nv|, so a 256-draw pilot samples zero-mean tails
    w = _out(SMALL["tiny_f32"], eps=0.3, pilot_min=256)
    x = synth.make_inputs(w)
    x["q"] = x["q"] * 2.0
    got, ref = check(w, inputs=x)
    ntail = 4096 - 4 - 64 - 128
    assert (got["budgets"] < ntail).any() and (got["budgets"] > 256).any(), got["budgets"]


@pytest.mark.parametrize("G", [1, 2, 8])
def test_group_sizes(G):
    w = _out(synth.scaled(W["gqa_32k"], max_ctx=5000, batch=2, num_q_heads=2 * G, num_kv_heads=2), eps=0.1)
    check(w, inputs=_coherent(w))


@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("f32", 128), ("f32", 64)])
def test_dtype_and_head_dim(dtype, d):
    w = _out(synth.scaled(W["gqa_32k"], max_ctx=3000, batch=2).replace(dtype=dtype, head_dim=d), eps=0.1)
    check(w, inputs=_coherent(w))


def test_zero_v_matches_the_denominator_budgets():
    w = SMALL["gqa"]
    x = synth.make_inputs(w)
    x["v_cache"] = torch.zeros_like(x["v_cache"])
    got_o, _ = check(_out(w), inputs=x)
    got_d, _ = check(w, inputs=x)
    for key in ("budgets", "head_need", "sel_count", "sel_idx"):
        assert np.array_equal(got_o[key], got_d[key]), key


def test_edge_lengths_paged():
    w = _out(synth.scaled(W["paged_sweep"], max_ctx=3000, min_ctx=3000, batch=8), eps=0.1)
    cpu = _coherent(w)
    cpu["seq_lens"] = torch.tensor([0, 5, 256, 257, 300, 1000, 2999, 3000], dtype=torch.int32)
    check(w, inputs=cpu)


def test_full_size_gqa_32k_every_unit():
    _full_check(_out(W["gqa_32k"], eps=0.5))


def test_unknown_guarantee_is_rejected():
    dev = _cuda()
    w = SMALL["tiny_f32"]
    x = {k: (v.to(dev) if hasattr(v, "to") else v) for k, v in synth.make_inputs(w).items()}
    dec = decoder_for(w)
    try:
        prm = params_for(w, x)
        prm.guarantee = 2
        o = dec.alloc_outputs(w.batch)
        rc = _abi.vattn_decode(dec.ctx, x["q"], x["k_cache"], x["v_cache"], x["page_table"],
                               x["seq_lens"], w.batch, prm, o["out"], o["sel_idx"], o["sel_count"],
                               o["budgets"], o["head_need"], check=False)
        assert rc == _abi.VATTN_EINVAL
    finally:
        dec.close()
