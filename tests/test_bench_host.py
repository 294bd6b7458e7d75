"""bench.py's host-side byte accounting (CPU only), against hand-counted cases."""
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from verified_sparse_attention_b200 import synth  # noqa: E402

GQA = synth.WORKLOADS["gqa_32k"]


def _counts(n, per_unit):
    return ({"seq_lens": torch.tensor(n, dtype=torch.int32)},
            {"sel_count": torch.tensor(per_unit, dtype=torch.int32)})


def test_score_and_gather_bytes_gqa_32k():
    # 8 sequences x 8 KV heads, middle 32768 - 128 - 128 rows of 256 B plus a 4-byte key
    x, res = _counts([32768] * 8, [[1239] * 8] * 8)
    b = bench.algorithmic_bytes(GQA, x, res)
    assert b["score_read"] == 8 * 8 * 32512 * 256
    assert b["key_write"] == 8 * 8 * 32512 * 4
    assert b["gather"] == 64 * 1239 * 2 * 256
    assert b["call"] == b["score_read"] + b["gather"]  # key writes are workspace, not KV reads


def test_proxy_score_bytes():
    # SparQ reads r = 32 of 128 dims per position from the dim-major copy; Loki 32 projected dims
    x, res = _counts([131072] * 4, [[100] * 8] * 4)
    for name in ("sparq_128k", "loki_64k"):
        w = synth.WORKLOADS[name].replace(max_ctx=131072, min_ctx=131072, batch=4)
        b = bench.algorithmic_bytes(w, x, res)
        mid = 131072 - w.sinks - w.window
        assert b["score_read"] == 4 * 8 * mid * 32 * 2, name


def test_output_guarantee_adds_one_v_read_of_if_and_the_pilot():
    # |I_f| = 128 sinks + floor(0.02 N) top-k + 128 window = 911, p = ceil(0.01 N) = 328
    x, res = _counts([32768] * 8, [[1239] * 8] * 8)
    call_d = bench.algorithmic_bytes(GQA, x, res)["call"]
    call_o = bench.algorithmic_bytes(GQA.replace(guarantee="output"), x, res)["call"]
    assert call_o - call_d == 8 * 8 * (911 + 328) * 256


def test_no_extra_read_without_a_pilot():
    # N = 400: middle 144, top-k 8, tail 136 > p = max(64, 4) = 64, so a pilot is drawn;
    # N = 300: middle 44, top-k 6, tail 38 <= 64, so the tail is taken whole without one
    x, res = _counts([400, 300], [[100] * 8] * 2)
    w = GQA.replace(batch=2)
    call_d = bench.algorithmic_bytes(w, x, res)["call"]
    call_o = bench.algorithmic_bytes(w.replace(guarantee="output"), x, res)["call"]
    n_if = 128 + (400 * 2) // 100 + 128
    assert call_o - call_d == 8 * (n_if + 64) * 256
