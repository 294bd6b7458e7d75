"""ctypes wrapper around the C oracle (oracle/vattn_oracle.c).

TEST INFRASTRUCTURE: only the tests, the package smoke check and the
benchmark's CPU-baseline leg import this module. The product package never
does, and shares no code with it.

Arrays are passed in the CUDA library's layouts (see `decode`). bf16 tensors
are passed as their raw 16-bit patterns.
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

F32, BF16 = 0, 1
EXACT, SPARQ, LOKI = 0, 1, 2
GUARANTEE_DENOMINATOR, GUARANTEE_OUTPUT = 0, 1
GUARANTEES = {"denominator": GUARANTEE_DENOMINATOR, "output": GUARANTEE_OUTPUT}
DTYPES = {"f32": F32, "bf16": BF16}
PROXIES = {"exact": EXACT, "sparq": SPARQ, "loki": LOKI}


class Problem(C.Structure):
    _fields_ = [
        ("batch", C.c_int), ("num_q_heads", C.c_int), ("num_kv_heads", C.c_int),
        ("head_dim", C.c_int), ("dtype", C.c_int),
        ("page_size", C.c_int), ("pages_per_seq", C.c_int), ("max_ctx", C.c_int),
        ("proxy", C.c_int), ("proxy_rank", C.c_int),
        ("sinks", C.c_int), ("window", C.c_int),
        ("topk_abs", C.c_int), ("topk_num", C.c_int), ("topk_den", C.c_int),
        ("pilot_min", C.c_int), ("pilot_num", C.c_int), ("pilot_den", C.c_int),
        ("eps", C.c_float), ("delta", C.c_float), ("seed", C.c_uint64),
        ("guarantee", C.c_int),
        ("topp_num", C.c_int), ("topp_den", C.c_int),
        ("batch_offset", C.c_int), ("head_offset", C.c_int),
    ]


_LIB = None


def lib(path=None):
    """Load (building first if stale) the oracle shared library."""
    global _LIB
    if path is not None:
        return _bind(C.CDLL(path))
    if _LIB is None:
        if _build.needs_build():
            _build.build()
        _LIB = _bind(C.CDLL(_build.OUT))
    return _LIB


def _bind(L):
    P = C.c_void_p
    L.orc_philox4x32_10.argtypes = [P, P, P]
    L.orc_philox4x32_10.restype = None
    L.orc_draw_word.argtypes = [C.c_uint64, C.c_uint32, C.c_uint32, C.c_uint32]
    L.orc_draw_word.restype = C.c_uint32
    L.orc_vexp.argtypes = [C.c_float]
    L.orc_vexp.restype = C.c_float
    L.orc_vexp_array.argtypes = [P, P, C.c_long]
    L.orc_vexp_array.restype = None
    L.orc_z.argtypes = [C.c_double]
    L.orc_z.restype = C.c_double
    L.orc_dot_chunked.argtypes = [P, P, C.c_int, C.c_int]
    L.orc_dot_chunked.restype = C.c_float
    L.orc_ord.argtypes = [C.c_float]
    L.orc_ord.restype = C.c_uint32
    L.orc_decode.argtypes = [C.POINTER(Problem)] + [P] * 8 + [P, C.c_int] + [P] * 7
    L.orc_decode.restype = C.c_int
    return L


def _np(x):
    """numpy view of a CPU array; bf16 torch tensors become uint16 bit patterns."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        import torch
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            return x.view(torch.int16).numpy().view(np.uint16)
        return x.numpy()
    return np.ascontiguousarray(x)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def philox(ctr, key, L=None):
    L = L or lib()
    c = np.asarray(ctr, dtype=np.uint32)
    k = np.asarray(key, dtype=np.uint32)
    o = np.zeros(4, dtype=np.uint32)
    L.orc_philox4x32_10(_ptr(c), _ptr(k), _ptr(o))
    return o


def draw_word(seed, b, h, t, L=None):
    return (L or lib()).orc_draw_word(seed, b, h, t)


def vexp(x, L=None):
    return (L or lib()).orc_vexp(float(x))


def vexp_array(x, L=None):
    x = np.ascontiguousarray(x, dtype=np.float32)
    y = np.empty_like(x)
    (L or lib()).orc_vexp_array(_ptr(x), _ptr(y), x.size)
    return y


def z_quantile(delta, L=None):
    return (L or lib()).orc_z(float(delta))


def dot_chunked(q, k, dtype, L=None):
    q = np.ascontiguousarray(q, dtype=np.float32)
    k = _np(k)
    return (L or lib()).orc_dot_chunked(_ptr(q), _ptr(k), q.shape[0], DTYPES[dtype])


def ord_key(f, L=None):
    return (L or lib()).orc_ord(float(f))


def make_problem(w, seed=None, eps=None, batch=None, guarantee=None, batch_offset=0, head_offset=0):
    """Problem struct from a workload description (verified_sparse_attention_b200.synth.Workload).

    `guarantee` ("denominator" or "output") overrides the workload's own; the
    offsets place a shard of a larger batch (its first sequence and KV head).
    """
    return Problem(
        batch=batch if batch is not None else w.batch, num_q_heads=w.num_q_heads,
        num_kv_heads=w.num_kv_heads, head_dim=w.head_dim, dtype=DTYPES[w.dtype],
        page_size=w.page_size, pages_per_seq=w.pages_per_seq, max_ctx=w.max_ctx,
        proxy=PROXIES[w.proxy], proxy_rank=w.proxy_rank, sinks=w.sinks, window=w.window,
        topk_abs=w.topk_abs, topk_num=w.topk_num, topk_den=w.topk_den,
        pilot_min=w.pilot_min, pilot_num=w.pilot_num, pilot_den=w.pilot_den,
        eps=w.eps if eps is None else eps, delta=w.delta,
        seed=w.seed if seed is None else seed,
        guarantee=GUARANTEES[guarantee or getattr(w, "guarantee", "denominator")],
        topp_num=getattr(w, "topp_num", 0), topp_den=getattr(w, "topp_den", 0),
        batch_offset=batch_offset, head_offset=head_offset)


def decode(problem, inputs, units=None, L=None):
    """Run the oracle on `inputs` (dict from synth.make_inputs, CPU tensors).

    Returns a dict of numpy arrays: out [B,Hq,d] float64, sel_idx [B,Hkv,max_ctx],
    sel_count [B,Hkv], budgets [B,Hkv], head_need [B,Hq], den_hat and ref_max
    [B,Hq] (estimated softmax denominator relative to exp(ref_max)). Only the
    listed units (b*Hkv + h) are written; other entries stay -1 / NaN.
    """
    L = L or lib()
    pr = problem
    B, Hq, Hkv, d = pr.batch, pr.num_q_heads, pr.num_kv_heads, pr.head_dim
    arrs = {k: _np(inputs.get(k)) for k in
            ("q", "k_cache", "v_cache", "k_t_cache", "k_proj_cache", "proj_basis",
             "page_table", "seq_lens")}
    if arrs["proj_basis"] is not None:
        arrs["proj_basis"] = np.ascontiguousarray(arrs["proj_basis"], dtype=np.float32)
    arrs["page_table"] = np.ascontiguousarray(arrs["page_table"], dtype=np.int32)
    arrs["seq_lens"] = np.ascontiguousarray(arrs["seq_lens"], dtype=np.int32)
    out = np.full((B, Hq, d), np.nan)
    sel_idx = np.full((B, Hkv, pr.max_ctx), -1, dtype=np.int32)
    sel_count = np.full((B, Hkv), -1, dtype=np.int32)
    budgets = np.full((B, Hkv), -1, dtype=np.int32)
    head_need = np.full((B, Hq), -1, dtype=np.int32)
    den_hat = np.full((B, Hq), np.nan)
    ref_max = np.full((B, Hq), np.nan)
    ul = None if units is None else np.ascontiguousarray(units, dtype=np.int32)
    rc = L.orc_decode(C.byref(pr), *[_ptr(arrs[k]) for k in
                                     ("q", "k_cache", "v_cache", "k_t_cache", "k_proj_cache",
                                      "proj_basis", "page_table", "seq_lens")],
                      _ptr(ul), 0 if ul is None else len(ul),
                      _ptr(out), _ptr(sel_idx), _ptr(sel_count), _ptr(budgets), _ptr(head_need),
                      _ptr(den_hat), _ptr(ref_max))
    if rc != 0:
        raise ValueError(f"oracle rejected the problem (code {rc})")
    return dict(out=out, sel_idx=sel_idx, sel_count=sel_count, budgets=budgets,
                head_need=head_need, den_hat=den_hat, ref_max=ref_max)
