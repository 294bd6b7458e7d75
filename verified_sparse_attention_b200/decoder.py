"""Convenience wrapper over the C ABI: one context plus its output buffers.

Marshalling only — every step runs in libvattn.so. Tensors are torch CUDA
tensors in the layouts of include/vattn.h.
"""
import torch

from . import _abi

_DTYPES = {torch.float32: _abi.VATTN_FP32, torch.bfloat16: _abi.VATTN_BF16}
_PROXIES = {"exact": _abi.VATTN_EXACT, "sparq": _abi.VATTN_SPARQ, "loki": _abi.VATTN_LOKI}
_GUARANTEES = {"denominator": _abi.VATTN_GUARANTEE_DENOMINATOR, "output": _abi.VATTN_GUARANTEE_OUTPUT}
# "host": k_cache and v_cache are page-locked host tensors (tensor.pin_memory())
_KV = {"device": _abi.VATTN_KV_DEVICE, "host": _abi.VATTN_KV_HOST}


class SparseDecoder:
    """A vattn context for fixed shapes (see vattn_config in include/vattn.h)."""

    def __init__(self, *, num_q_heads, num_kv_heads, head_dim, dtype, page_size, max_batch,
                 max_ctx, proxy="exact", proxy_rank=0, device=None, kv_location="device"):
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.num_q_heads, self.num_kv_heads, self.head_dim = num_q_heads, num_kv_heads, head_dim
        self.max_batch, self.max_ctx, self.page_size = max_batch, max_ctx, page_size
        self.proxy = proxy
        self.dtype = dtype
        cfg = _abi.vattn_config(num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
                                head_dim=head_dim, dtype=_DTYPES[dtype], page_size=page_size,
                                max_batch=max_batch, max_ctx=max_ctx, proxy=_PROXIES[proxy],
                                proxy_rank=proxy_rank, kv_location=_KV[kv_location])
        with torch.cuda.device(self.device):
            self.ctx = _abi.vattn_create(cfg)

    def alloc_outputs(self, batch):
        dev = self.device
        return dict(
            out=torch.empty((batch, self.num_q_heads, self.head_dim), dtype=torch.float32, device=dev),
            sel_idx=torch.empty((batch, self.num_kv_heads, self.max_ctx), dtype=torch.int32, device=dev),
            sel_count=torch.empty((batch, self.num_kv_heads), dtype=torch.int32, device=dev),
            budgets=torch.empty((batch, self.num_kv_heads), dtype=torch.int32, device=dev),
            head_need=torch.empty((batch, self.num_q_heads), dtype=torch.int32, device=dev))

    @staticmethod
    def make_params(*, sinks, window, topk_abs=0, topk_num=0, topk_den=0, pilot_min=64,
                    pilot_num=0, pilot_den=0, eps, delta, seed, num_pages, k_t_cache=None,
                    k_proj_cache=None, proj_basis=None, guarantee="denominator", topp_num=0,
                    topp_den=0, batch_offset=0, head_offset=0):
        return _abi.vattn_params(
            sinks=sinks, window=window, topk_abs=topk_abs, topk_num=topk_num, topk_den=topk_den,
            pilot_min=pilot_min, pilot_num=pilot_num, pilot_den=pilot_den, eps=eps, delta=delta,
            seed=seed, num_pages=num_pages,
            k_t_cache=None if k_t_cache is None else k_t_cache.data_ptr(),
            k_proj_cache=None if k_proj_cache is None else k_proj_cache.data_ptr(),
            proj_basis=None if proj_basis is None else proj_basis.data_ptr(),
            guarantee=_GUARANTEES[guarantee], topp_num=topp_num, topp_den=topp_den,
            batch_offset=batch_offset, head_offset=head_offset)

    def decode(self, q, k_cache, v_cache, page_table, seq_lens, params, outputs=None, stream=None):
        batch = q.shape[0]
        o = outputs if outputs is not None else self.alloc_outputs(batch)
        _abi.vattn_decode(self.ctx, q, k_cache, v_cache, page_table, seq_lens, batch, params,
                          o["out"], o["sel_idx"], o["sel_count"], o["budgets"], o["head_need"],
                          stream=stream)
        return o

    def dense(self, q, k_cache, v_cache, page_table, seq_lens, num_pages, out=None, stream=None):
        batch = q.shape[0]
        if out is None:
            out = torch.empty((batch, self.num_q_heads, self.head_dim), dtype=torch.float32,
                              device=self.device)
        _abi.vattn_dense_decode(self.ctx, q, k_cache, v_cache, page_table, seq_lens, batch,
                                num_pages, out, stream=stream)
        return out

    def last_error(self, sync=True):
        return _abi.vattn_last_error(self.ctx, sync)

    def close(self):
        if getattr(self, "ctx", None):
            _abi.vattn_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def decoder_for(w, device=None, max_batch=None, kv_location="device"):
    """A SparseDecoder shaped for a synthetic workload description (synth.Workload)."""
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    return SparseDecoder(num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads,
                         head_dim=w.head_dim, dtype=dt, page_size=w.page_size,
                         max_batch=w.batch if max_batch is None else max_batch, max_ctx=w.max_ctx,
                         proxy=w.proxy, proxy_rank=w.proxy_rank, device=device,
                         kv_location=kv_location)


def params_for(w, inputs, eps=None, seed=None, guarantee=None, batch_offset=0, head_offset=0):
    """vattn_params of a synthetic workload with its drawn inputs (device tensors); the
    offsets place a shard of a larger batch."""
    return SparseDecoder.make_params(
        sinks=w.sinks, window=w.window, topk_abs=w.topk_abs, topk_num=w.topk_num,
        topk_den=w.topk_den, pilot_min=w.pilot_min, pilot_num=w.pilot_num, pilot_den=w.pilot_den,
        eps=w.eps if eps is None else eps, delta=w.delta, seed=w.seed if seed is None else seed,
        num_pages=int(inputs["num_pages"]), k_t_cache=inputs.get("k_t_cache"),
        k_proj_cache=inputs.get("k_proj_cache"), proj_basis=inputs.get("proj_basis"),
        guarantee=guarantee or w.guarantee, topp_num=w.topp_num, topp_den=w.topp_den,
        batch_offset=batch_offset, head_offset=head_offset)
