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
    score, call = bench.algorithmic_bytes(GQA, x, res)
    assert score == 8 * 8 * 32512 * (256 + 4)
    assert call == score + 64 * 1239 * 2 * 256


def test_output_guarantee_adds_one_v_read_of_if_and_the_pilot():
    # |I_f| = 128 sinks + floor(0.02 N) top-k + 128 window = 911, p = ceil(0.01 N) = 328
    x, res = _counts([32768] * 8, [[1239] * 8] * 8)
    _, call_d = bench.algorithmic_bytes(GQA, x, res)
    _, call_o = bench.algorithmic_bytes(GQA.replace(guarantee="output"), x, res)
    assert call_o - call_d == 8 * 8 * (911 + 328) * 256


def test_no_extra_read_without_a_pilot():
    # N = 400: middle 144, top-k 8, tail 136 > p = max(64, 4) = 64, so a pilot is drawn;
    # N = 300: middle 44, top-k 6, tail 38 <= 64, so the tail is taken whole without one
    x, res = _counts([400, 300], [[100] * 8] * 2)
    w = GQA.replace(batch=2)
    _, call_d = bench.algorithmic_bytes(w, x, res)
    _, call_o = bench.algorithmic_bytes(w.replace(guarantee="output"), x, res)
    n_if = 128 + (400 * 2) // 100 + 128
    assert call_o - call_d == 8 * (n_if + 64) * 256
