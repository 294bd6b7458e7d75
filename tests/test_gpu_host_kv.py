"""KV cache hosted in page-locked host memory (vattn_config.kv_location = host).

The vAttention page reports speedups when the KV cache lives on the CPU
("Performance and Efficiency"): the method reads only the rows it selects. Here
the K and V caches are pinned host tensors; q, the page table, the lengths and
the SparQ / Loki proxy caches stay on the GPU. The index sets, budgets and
per-head sizes must match the oracle bit for bit, and the outputs stay within
the usual tolerance, exactly as with device-resident caches.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import dense_attention, rel_err_rows
from tests.test_gpu_parity import SMALL, TOL, W, _cuda, compare
from verified_sparse_attention_b200 import _abi, synth
from verified_sparse_attention_b200.decoder import decoder_for, params_for

pytestmark = pytest.mark.gpu


def _host_split(cpu, dev):
    """Device copies of everything but the K and V caches, which stay pinned on the host."""
    x = {k: (v.to(dev) if hasattr(v, "to") and k not in ("k_cache", "v_cache") else v) for k, v in cpu.items()}
    x["k_cache"] = cpu["k_cache"].pin_memory()
    x["v_cache"] = cpu["v_cache"].pin_memory()
    return x


def _run_host(w, x):
    dec = decoder_for(w, kv_location="host")
    try:
        res = dec.decode(x["q"], x["k_cache"], x["v_cache"], x["page_table"], x["seq_lens"],
                         params_for(w, x))
        torch.cuda.synchronize()
        err = dec.last_error()
        return {k: v.cpu().numpy() for k, v in res.items()}, err
    finally:
        dec.close()


@pytest.mark.parametrize("name", ["tiny_f32", "gqa", "sparq", "loki", "paged"])
def test_parity_host_resident_caches(name):
    w = SMALL[name]
    dev = _cuda()
    cpu = synth.make_inputs(w)
    got, err = _run_host(w, _host_split(cpu, dev))
    assert err == 0
    ref = oracle.decode(oracle.make_problem(w), cpu)
    compare(w, got, ref, range(w.units))


def test_parity_host_resident_caches_top_p_and_output_guarantee():
    dev = _cuda()
    w = SMALL["gqa"].replace(topp_num=9, topp_den=10)
    cpu = synth.make_inputs(w)
    got, err = _run_host(w, _host_split(cpu, dev))
    assert err == 0
    compare(w, got, oracle.decode(oracle.make_problem(w), cpu), range(w.units))
    w = SMALL["gqa"].replace(guarantee="output", eps=0.3)
    cpu = synth.make_inputs(w)
    cpu["v_cache"] = cpu["v_cache"] + 1.0
    got, err = _run_host(w, _host_split(cpu, dev))
    assert err == 0
    compare(w, got, oracle.decode(oracle.make_problem(w), cpu), range(w.units))


def test_full_size_loki_64k_every_unit():
    w = W["loki_64k"]
    dev = _cuda()
    xd = synth.make_inputs(w, device=dev)
    cpu = {k: (v.cpu() if hasattr(v, "cpu") else v) for k, v in xd.items()}
    x = dict(xd, k_cache=cpu["k_cache"].pin_memory(), v_cache=cpu["v_cache"].pin_memory())
    del xd
    torch.cuda.empty_cache()
    got, err = _run_host(w, x)
    assert err == 0
    units = list(range(w.units))
    compare(w, got, oracle.decode(oracle.make_problem(w), cpu, units=units), units)


def test_dense_decode_over_host_resident_caches():
    w = SMALL["paged"]
    dev = _cuda()
    cpu = synth.make_inputs(w)
    x = _host_split(cpu, dev)
    dec = decoder_for(w, kv_location="host")
    try:
        out = dec.dense(x["q"], x["k_cache"], x["v_cache"], x["page_table"], x["seq_lens"],
                        x["num_pages"]).cpu().numpy()
        assert dec.last_error() == 0
    finally:
        dec.close()
    for b in range(w.batch):
        for hq in range(0, w.num_q_heads, 5):
            assert rel_err_rows(out[b, hq], dense_attention(cpu, w, b, hq)) <= TOL[w.dtype]


def test_static_dense_decode_over_host_resident_caches():
    w = SMALL["gqa"]
    dev = _cuda()
    cpu = synth.make_inputs(w)
    x = _host_split(cpu, dev)
    cfg = _abi.vattn_config(num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads,
                            head_dim=w.head_dim, dtype=_abi.VATTN_BF16, page_size=w.page_size,
                            max_batch=w.batch, max_ctx=w.max_ctx, proxy=_abi.VATTN_EXACT,
                            proxy_rank=0, kv_location=_abi.VATTN_KV_HOST)
    out = torch.full((w.batch, w.num_q_heads, w.head_dim), float("nan"), device=dev)
    _abi.vattn_dense_decode_static(cfg, x["q"], x["k_cache"], x["v_cache"], x["page_table"],
                                   x["seq_lens"], w.batch, x["num_pages"], out)
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    for b in range(w.batch):
        for hq in range(0, w.num_q_heads, 7):
            assert rel_err_rows(out[b, hq], dense_attention(cpu, w, b, hq)) <= TOL[w.dtype]


def test_caches_that_are_not_page_locked_host_memory_are_refused():
    w = SMALL["tiny_f32"]
    dev = _cuda()
    cpu = synth.make_inputs(w)
    x = _host_split(cpu, dev)
    dec = decoder_for(w, kv_location="host")
    try:
        o = dec.alloc_outputs(w.batch)
        prm = params_for(w, x)
        for k_cache in (cpu["k_cache"].clone(), cpu["k_cache"].to(dev)):  # pageable host; device
            rc = _abi.vattn_decode(dec.ctx, x["q"], k_cache, x["v_cache"], x["page_table"],
                                   x["seq_lens"], w.batch, prm, o["out"], o["sel_idx"],
                                   o["sel_count"], o["budgets"], o["head_need"], check=False)
            assert rc == _abi.VATTN_EINVAL
    finally:
        dec.close()
