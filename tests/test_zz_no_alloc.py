"""vattn_dense_decode_static: the dense decode that allocates nothing.

Its scratch is one fixed device array shared by every call on a device, so
the GPU test makes two calls in a row on different inputs (the second one
finds the first one's partial results in the array) and compares each with
vattn_dense_decode, the context-based entry point, on the same inputs.
"""
import numpy as np
import pytest
import torch

from tests.helpers import dense_attention, rel_err_rows
from verified_sparse_attention_b200 import _abi, synth

TOL = {"bf16": 2e-3, "f32": 1e-5}
_DT = {"bf16": _abi.VATTN_BF16, "f32": _abi.VATTN_FP32}


def _config(w, max_batch=None):
    return _abi.vattn_config(num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads,
                             head_dim=w.head_dim, dtype=_DT[w.dtype], page_size=w.page_size,
                             max_batch=max_batch or w.batch, max_ctx=w.max_ctx,
                             proxy=_abi.VATTN_EXACT, proxy_rank=0)


def test_oversize_call_is_refused_before_touching_the_device():
    # 2048 sequences x 32 query heads x (128 + 2) floats = 34 MB > the 8 MiB array;
    # the pointers are never dereferenced because the size check comes first
    w = synth.WORKLOADS["gqa_32k"]
    cfg = _config(w, max_batch=4096)
    fake = 1 << 20
    rc = _abi.vattn_dense_decode_static(cfg, fake, fake, fake, fake, fake, 2048, 1, fake,
                                        stream=0, check=False)
    assert rc == _abi.VATTN_ESCRATCH
    assert "8 MiB" in _abi.vattn_strerror(rc)
    bad = _config(w)
    bad.head_dim = 96
    assert _abi.vattn_dense_decode_static(bad, fake, fake, fake, fake, fake, 1, 1, fake,
                                          stream=0, check=False) == _abi.VATTN_EINVAL


def _dense_with_context(w, x):
    ctx = _abi.vattn_create(_config(w))
    try:
        out = torch.empty((w.batch, w.num_q_heads, w.head_dim), dtype=torch.float32, device="cuda")
        _abi.vattn_dense_decode(ctx, x["q"], x["k_cache"], x["v_cache"], x["page_table"],
                                x["seq_lens"], w.batch, x["num_pages"], out)
        torch.cuda.synchronize()
        assert _abi.vattn_last_error(ctx) == 0
        return out.cpu().numpy()
    finally:
        _abi.vattn_destroy(ctx)


def _dense_static(w, x):
    out = torch.full((w.batch, w.num_q_heads, w.head_dim), float("nan"), dtype=torch.float32,
                     device="cuda")
    _abi.vattn_dense_decode_static(_config(w), x["q"], x["k_cache"], x["v_cache"],
                                   x["page_table"], x["seq_lens"], w.batch, x["num_pages"], out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.gpu
@pytest.mark.parametrize("first,second", [
    # contiguous bf16 cache, 4 query heads per KV head, then a paged cache
    (dict(name="gqa_32k", max_ctx=9000, min_ctx=5000, batch=3, data_seed=11),
     dict(name="paged_sweep", max_ctx=7000, min_ctx=3000, batch=4, data_seed=12)),
    # fp32: one query head per KV head at d 64, then eight per KV head at d 128
    (dict(name="tiny_f32", max_ctx=4096, min_ctx=1000, batch=3, data_seed=13),
     dict(name="tiny_f32", max_ctx=3000, min_ctx=2000, batch=2, data_seed=14, num_q_heads=16,
          num_kv_heads=2, head_dim=128)),
])
def test_two_calls_in_a_row_match_the_context_entry(first, second):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    for spec in (first, second):
        spec = dict(spec)
        w = synth.scaled(synth.WORKLOADS[spec.pop("name")], **spec)
        cpu = synth.make_inputs(w)
        x = {k: (v.to("cuda") if hasattr(v, "to") else v) for k, v in cpu.items()}
        ref = _dense_with_context(w, x)
        got = _dense_static(w, x)
        assert np.isfinite(got).all()
        err = rel_err_rows(got.reshape(-1, w.head_dim), ref.reshape(-1, w.head_dim))
        assert err.max() <= TOL[w.dtype], (w.name, float(err.max()))
        # and against float64 dense attention computed from the caches
        for b in range(w.batch):
            for hq in range(0, w.num_q_heads, max(1, w.num_q_heads // 4)):
                e = rel_err_rows(got[b, hq], dense_attention(cpu, w, b, hq))
                assert e <= TOL[w.dtype], (w.name, b, hq, float(e))


@pytest.mark.gpu
def test_bad_sequences_give_zero_rows_and_leave_the_others_alone():
    # a page id past the pool, a length above max_ctx and an empty sequence: their
    # rows are exactly 0 (there is no error word without a context); the other
    # sequences match the context entry point on the same inputs
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = synth.scaled(synth.WORKLOADS["paged_sweep"], max_ctx=3000, min_ctx=1500, batch=5,
                     data_seed=15)
    cpu = synth.make_inputs(w)
    cpu["page_table"][1, 7] = cpu["num_pages"] + 3
    cpu["seq_lens"][2] = w.max_ctx + 1
    cpu["seq_lens"][3] = 0
    x = {k: (v.to("cuda") if hasattr(v, "to") else v) for k, v in cpu.items()}
    for _ in range(2):  # the second call finds the first one's records in the array
        got = _dense_static(w, x)
        assert np.all(got[1:4] == 0.0)
        ref = _dense_with_context_any_error(w, x)
        for b in (0, 4):
            err = rel_err_rows(got[b], ref[b])
            assert err.max() <= TOL[w.dtype], (b, float(err.max()))


def _dense_with_context_any_error(w, x):
    ctx = _abi.vattn_create(_config(w))
    try:
        out = torch.empty((w.batch, w.num_q_heads, w.head_dim), dtype=torch.float32, device="cuda")
        _abi.vattn_dense_decode(ctx, x["q"], x["k_cache"], x["v_cache"], x["page_table"],
                                x["seq_lens"], w.batch, x["num_pages"], out)
        torch.cuda.synchronize()
        assert _abi.vattn_last_error(ctx) != 0  # the context entry point reports the bad rows
        return out.cpu().numpy()
    finally:
        _abi.vattn_destroy(ctx)
