"""Brute-force helpers for the tests (numpy, float64). No decode-step logic."""
import math

import numpy as np
import torch


def to_f64(t):
    return t.detach().cpu().float().double().numpy() if hasattr(t, "detach") else np.asarray(t, np.float64)


def logical_rows(inputs, w, b, h, key="k_cache"):
    """Rows [0, N_b) of sequence b, KV head h, gathered through the page table (float64)."""
    n = int(inputs["seq_lens"][b])
    ps = w.page_size
    pt = inputs["page_table"][b].cpu().numpy()
    cache = inputs[key]
    rows = []
    for p in range(-(-n // ps)):
        rows.append(cache[int(pt[p]), h].float().double().cpu().numpy())
    if not rows:
        return np.zeros((0, cache.shape[-1]))
    return np.concatenate(rows, 0)[:n]


def exact_scores(inputs, w, b, hq):
    """float64 q_h . k_j / sqrt(d) over all positions of sequence b."""
    G = w.group
    K = logical_rows(inputs, w, b, hq // G)
    q = to_f64(inputs["q"][b, hq])
    return K @ q / math.sqrt(w.head_dim)


def dense_attention(inputs, w, b, hq):
    """float64 softmax attention of query head hq over all positions of sequence b."""
    s = exact_scores(inputs, w, b, hq)
    V = logical_rows(inputs, w, b, hq // w.group, "v_cache")
    if len(s) == 0:
        return np.zeros(w.head_dim)
    e = np.exp(s - s.max())
    return (e[:, None] * V).sum(0) / e.sum()


def rel_err_rows(a, ref):
    """max |a - ref| / max |ref| per row (last axis), as an array over rows."""
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    num = np.abs(a - ref).max(-1)
    den = np.maximum(np.abs(ref).max(-1), 1e-30)
    return num / den


def regions(w, n):
    """(s1, wst, mlen, k, p) for a sequence of length n — stated from the workload's parameters."""
    s1 = min(w.sinks, n)
    wst = max(n - w.window, s1)
    mlen = wst - s1
    kb = w.topk_abs if w.topk_den == 0 else (n * w.topk_num) // w.topk_den
    p = w.pilot_min if w.pilot_den == 0 else max(w.pilot_min, -(-n * w.pilot_num // w.pilot_den))
    return s1, wst, mlen, min(kb, mlen), p
