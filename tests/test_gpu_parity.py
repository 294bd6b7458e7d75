"""CUDA path (through the C ABI) against the oracle, element by element.

Selected indices, counts, budgets and per-head sample sizes must match bit for
bit; outputs within max|o - o_ref| / max|o_ref| per (sequence, query head) row
of 2e-3 for bf16 caches and 1e-5 for fp32 caches.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import dense_attention, rel_err_rows
from verified_sparse_attention_b200 import _abi, synth
from verified_sparse_attention_b200.decoder import decoder_for, params_for

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-3, "f32": 1e-5}
W = synth.WORKLOADS


def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def _to(inputs, dev):
    return {k: (v.to(dev) if hasattr(v, "to") else v) for k, v in inputs.items()}


def run_gpu(w, inputs_dev, eps=None, seed=None):
    dec = decoder_for(w)
    try:
        res = dec.decode(inputs_dev["q"], inputs_dev["k_cache"], inputs_dev["v_cache"],
                         inputs_dev["page_table"], inputs_dev["seq_lens"],
                         params_for(w, inputs_dev, eps=eps, seed=seed))
        torch.cuda.synchronize()
        err = dec.last_error()
        return {k: v.cpu().numpy() for k, v in res.items()}, err
    finally:
        dec.close()


def compare(w, got, ref, units):
    Hkv, G = w.num_kv_heads, w.group
    for u in units:
        b, h = divmod(int(u), Hkv)
        cnt = int(ref["sel_count"][b, h])
        assert int(got["sel_count"][b, h]) == cnt, (u, got["sel_count"][b, h], cnt)
        assert int(got["budgets"][b, h]) == int(ref["budgets"][b, h]), u
        assert np.array_equal(got["head_need"][b, h * G:(h + 1) * G],
                              ref["head_need"][b, h * G:(h + 1) * G]), u
        assert np.array_equal(got["sel_idx"][b, h, :cnt], ref["sel_idx"][b, h, :cnt]), u
        err = rel_err_rows(got["out"][b, h * G:(h + 1) * G], ref["out"][b, h * G:(h + 1) * G])
        assert err.max() <= TOL[w.dtype], (u, err.max())


def check(w, eps=None, seed=None, units=None, inputs=None):
    dev = _cuda()
    cpu = synth.make_inputs(w) if inputs is None else inputs
    got, err = run_gpu(w, _to(cpu, dev), eps=eps, seed=seed)
    assert err == 0
    ref = oracle.decode(oracle.make_problem(w, eps=eps, seed=seed), cpu, units=units)
    compare(w, got, ref, range(w.units) if units is None else units)
    return got, ref


# ------------------------------------------------------------ reduced sizes, all units
SMALL = {
    "tiny_f32": W["tiny_f32"],
    "tiny_f32_ragged": synth.scaled(W["tiny_f32"], max_ctx=4001),
    "gqa": synth.scaled(W["gqa_32k"], max_ctx=9000, batch=2),
    "sparq": synth.scaled(W["sparq_128k"], max_ctx=10000, batch=2),
    "loki": synth.scaled(W["loki_64k"], max_ctx=7000, batch=2),
    "paged": synth.scaled(W["paged_sweep"], max_ctx=9000, min_ctx=3000, batch=4),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_parity_reduced(name):
    check(SMALL[name])


@pytest.mark.parametrize("eps", synth.PAGED_EPS_SWEEP)
def test_parity_paged_eps_sweep_reduced(eps):
    check(SMALL["paged"], eps=eps)


@pytest.mark.parametrize("seed", [1, 2, 0xFFFFFFFFFFFFFFFF])
def test_parity_seeds(seed):
    check(SMALL["gqa"], seed=seed)


# ------------------------------------------------------------ edge cases
def test_edge_lengths_paged():
    # empty, shorter than the sinks, middle exactly empty, exhausted, page-ragged
    w = synth.scaled(W["paged_sweep"], max_ctx=3000, min_ctx=3000, batch=8)
    cpu = synth.make_inputs(w)
    lens = [0, 5, 128 + 128, 128 + 128 + 1, 300, 1000, 2999, 3000]
    cpu["seq_lens"] = torch.tensor(lens, dtype=torch.int32)
    check(w, inputs=cpu)


@pytest.mark.parametrize("G", [1, 2, 8])
def test_group_sizes(G):
    w = synth.scaled(W["gqa_32k"], max_ctx=5000, batch=2, num_q_heads=2 * G, num_kv_heads=2)
    check(w)


@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("f32", 128), ("f32", 64), ("bf16", 128)])
def test_dtype_and_head_dim(dtype, d):
    w = synth.scaled(W["gqa_32k"], max_ctx=3000, batch=2).replace(dtype=dtype, head_dim=d)
    check(w)


def test_long_max_ctx_streams_the_keys():
    # a context bound whose keys do not fit one CTA's shared memory selects with
    # k_topk, which streams the keys from L2
    small = synth.scaled(W["gqa_32k"], max_ctx=9000, batch=1, num_q_heads=8, num_kv_heads=2)
    cpu = synth.make_inputs(small)
    w = small.replace(max_ctx=600000, min_ctx=600000)      # same page size, longer bound
    pad = torch.full((1, w.pages_per_seq - cpu["page_table"].shape[1]), -1, dtype=torch.int32)
    cpu["page_table"] = torch.cat([cpu["page_table"], pad], 1)
    check(w, inputs=cpu)


@pytest.mark.parametrize("case", ["equal_scores", "k_above_list_space", "planted"])
def test_streamed_select_at_long_context(case):
    # k_topk (middles longer than one CTA's shared memory): the single ordered pass,
    # and its fallback when a list would overflow (every score equal puts every key
    # in one bin; k above the space for the keys above the cut bin)
    w = synth.scaled(W["gqa_32k"], max_ctx=50000, batch=1, num_q_heads=8, num_kv_heads=2)
    if case == "k_above_list_space":
        w = w.replace(topk_num=0, topk_den=0, topk_abs=9000)
    cpu = synth.make_inputs(w)
    if case == "equal_scores":
        cpu["q"].zero_()
    check(w, inputs=cpu)


def test_no_topk_and_large_topk():
    base = synth.scaled(W["tiny_f32"], max_ctx=2000)
    check(base.replace(topk_abs=0))
    check(base.replace(topk_abs=1900))          # top-k swallows the middle


def test_ties_at_the_threshold():
    w = synth.scaled(W["tiny_f32"], max_ctx=3000).replace(topk_abs=50)
    cpu = synth.make_inputs(w)
    for h in range(4):
        qh = cpu["q"][0, h]
        row = 5.0 * qh / qh.norm()
        for p in range(200, 2800, 23):                 # 113 identical rows, 50 to take
            cpu["k_cache"][0, h, p] = row
    check(w, inputs=cpu)


def test_all_scores_equal():
    w = synth.scaled(W["gqa_32k"], max_ctx=6000, batch=1)
    cpu = synth.make_inputs(w)
    cpu["q"].zero_()
    check(w, inputs=cpu)


def test_eps_tiny_is_dense():
    w = SMALL["gqa"]
    dev = _cuda()
    cpu = synth.make_inputs(w)
    got, err = run_gpu(w, _to(cpu, dev), eps=1e-7)
    assert err == 0
    for b in range(w.batch):
        for hq in range(w.num_q_heads):
            ref = dense_attention(cpu, w, b, hq)
            assert rel_err_rows(got["out"][b, hq], ref) <= TOL[w.dtype]


def test_dense_decode_kernel():
    w = SMALL["paged"]
    dev = _cuda()
    cpu = synth.make_inputs(w)
    x = _to(cpu, dev)
    dec = decoder_for(w)
    try:
        out = dec.dense(x["q"], x["k_cache"], x["v_cache"], x["page_table"], x["seq_lens"],
                        x["num_pages"]).cpu().numpy()
        assert dec.last_error() == 0
    finally:
        dec.close()
    for b in range(w.batch):
        for hq in range(0, w.num_q_heads, 3):
            ref = dense_attention(cpu, w, b, hq)
            assert rel_err_rows(out[b, hq], ref) <= TOL[w.dtype]


def test_deterministic_bits():
    w = SMALL["paged"]
    dev = _cuda()
    x = _to(synth.make_inputs(w), dev)
    a, _ = run_gpu(w, x)
    b, _ = run_gpu(w, x)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


# ------------------------------------------------------------ device error word
def test_bad_page_sets_error_and_empties_the_sequence():
    w = synth.scaled(W["paged_sweep"], max_ctx=2000, min_ctx=1500, batch=3)
    dev = _cuda()
    cpu = synth.make_inputs(w)
    cpu["page_table"][1, 3] = 10 ** 6            # out of range: caught by the kernel's check
    got, err = run_gpu(w, _to(cpu, dev))
    assert err & _abi.VATTN_DEV_BAD_PAGE
    assert np.all(got["out"][1] == 0) and np.all(got["sel_count"][1] == 0)
    # the other sequences are untouched by the bad one
    ref = oracle.decode(oracle.make_problem(w), cpu, units=[0, 2 * w.num_kv_heads])
    compare(w, got, ref, [0, 2 * w.num_kv_heads])


def test_bad_length_sets_error():
    w = synth.scaled(W["tiny_f32"], max_ctx=1000)
    dev = _cuda()
    cpu = synth.make_inputs(w)
    cpu["seq_lens"][0] = 5000                    # above max_ctx
    got, err = run_gpu(w, _to(cpu, dev))
    assert err & _abi.VATTN_DEV_BAD_SEQLEN
    assert np.all(got["out"] == 0)


def test_context_reuse_with_fewer_items_than_record_producers():
    # one context, two calls: the first gathers more items than the gathers have
    # record producers (every producer writes records), the second fewer (most
    # producers own no item and write no record), so the second call must read
    # only the records it wrote, not the first call's left in the workspace
    w = SMALL["tiny_f32"]
    dev = _cuda()
    cpu = synth.make_inputs(w)
    x = _to(cpu, dev)
    dec = decoder_for(w)
    try:
        for topk in (1500, w.topk_abs):
            wc = w.replace(topk_abs=topk)
            res = dec.decode(x["q"], x["k_cache"], x["v_cache"], x["page_table"], x["seq_lens"],
                             params_for(wc, x))
            torch.cuda.synchronize()
            assert dec.last_error() == 0
            got = {k: v.cpu().numpy() for k, v in res.items()}
            compare(wc, got, oracle.decode(oracle.make_problem(wc), cpu), range(w.units))
    finally:
        dec.close()


def test_bounded_wait_runs_out_and_reports_a_timeout():
    # a wait on a barrier that no copy completes: the kernel gives up after its
    # limit, sets VATTN_DEV_TIMEOUT and returns; the context stays usable
    w = SMALL["tiny_f32"]
    dev = _cuda()
    dec = decoder_for(w)
    try:
        assert dec.last_error() == 0
        for tries in (1, 1000):
            _abi.vattn_check_bounded_wait(dec.ctx, tries)
            assert dec.last_error() == _abi.VATTN_DEV_TIMEOUT  # read and cleared
            assert dec.last_error() == 0
        assert _abi.vattn_check_bounded_wait(dec.ctx, 0, check=False) == _abi.VATTN_EINVAL
        assert _abi.vattn_check_bounded_wait(dec.ctx, (1 << 20) + 1, check=False) == _abi.VATTN_EINVAL
    finally:
        dec.close()
    check(w)  # a decode on the same device afterwards is still exact


def test_host_argument_checks():
    w = SMALL["tiny_f32"]
    dev = _cuda()
    x = _to(synth.make_inputs(w), dev)
    dec = decoder_for(w)
    try:
        o = dec.alloc_outputs(w.batch)
        for kw in [dict(eps=0.0), dict(eps=-1.0), dict(delta=0.0), dict(delta=1.0)]:
            p = params_for(w, x)
            for k, v in kw.items():
                setattr(p, k, v)
            rc = _abi.vattn_decode(dec.ctx, x["q"], x["k_cache"], x["v_cache"], x["page_table"],
                                   x["seq_lens"], w.batch, p, o["out"], o["sel_idx"],
                                   o["sel_count"], o["budgets"], o["head_need"], check=False)
            assert rc == _abi.VATTN_EINVAL, kw
        p = params_for(w, x)
        p.pilot_min = 1
        assert _abi.vattn_decode(dec.ctx, x["q"], x["k_cache"], x["v_cache"], x["page_table"],
                                 x["seq_lens"], w.batch, p, o["out"], o["sel_idx"], o["sel_count"],
                                 o["budgets"], o["head_need"], check=False) == _abi.VATTN_EINVAL
        p = params_for(w, x)
        assert _abi.vattn_decode(dec.ctx, x["q"], x["k_cache"], x["v_cache"], x["page_table"],
                                 x["seq_lens"], w.batch + 1, p, o["out"], o["sel_idx"],
                                 o["sel_count"], o["budgets"], o["head_need"],
                                 check=False) == _abi.VATTN_EINVAL
    finally:
        dec.close()
    sq = synth.scaled(W["sparq_128k"], max_ctx=512, batch=1)
    dec = decoder_for(sq)
    try:
        xs = _to(synth.make_inputs(sq), dev)
        p = params_for(sq, xs)
        p.k_t_cache = None
        o = dec.alloc_outputs(1)
        assert _abi.vattn_decode(dec.ctx, xs["q"], xs["k_cache"], xs["v_cache"], xs["page_table"],
                                 xs["seq_lens"], 1, p, o["out"], o["sel_idx"], o["sel_count"],
                                 o["budgets"], o["head_need"], check=False) == _abi.VATTN_EINVAL
    finally:
        dec.close()


# ------------------------------------------------------------ full sizes, sampled units
FULL = ["gqa_32k", "sparq_128k", "loki_64k", "paged_sweep"]


def _full_check(w, eps=None):
    """Every unit of a full-size call against the oracle (a second or a few of
    oracle time per workload), plus bounds that hold for every unit."""
    dev = _cuda()
    x = synth.make_inputs(w, device=dev)
    got, err = run_gpu(w, x, eps=eps)
    assert err == 0
    units = list(range(w.units))
    cpu = {k: (v.cpu() if hasattr(v, "cpu") else v) for k, v in x.items()}
    del x
    torch.cuda.empty_cache()
    ref = oracle.decode(oracle.make_problem(w, eps=eps), cpu, units=units)
    compare(w, got, ref, units)
    # properties that hold for every unit
    Hkv = w.num_kv_heads
    n = cpu["seq_lens"].numpy()
    for u in range(w.units):
        b, h = divmod(u, Hkv)
        cnt = got["sel_count"][b, h]
        s = got["sel_idx"][b, h, :cnt]
        assert cnt <= n[b] and np.all((s >= 0) & (s < n[b]))


@pytest.mark.parametrize("name", FULL)
def test_parity_full_size_every_unit(name):
    _full_check(W[name])


def test_parity_full_tiny():
    check(W["tiny_f32"])


@pytest.mark.parametrize("eps", [0.01, 0.2])
def test_parity_full_paged_eps(eps):
    _full_check(W["paged_sweep"], eps=eps)
