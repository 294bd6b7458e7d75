"""Thin ctypes binding of the C ABI in include/vattn.h (argument marshalling only).

Every step of the decode runs in libvattn.so's CUDA kernels. Loading fails
loudly if the library has not been built: there is no fallback path.
Tensors are passed by data pointer; they must already live on the CUDA
device of the context (torch is used for device memory and streams only).
"""
import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvattn.so")

VATTN_FP32, VATTN_BF16 = 0, 1
VATTN_EXACT, VATTN_SPARQ, VATTN_LOKI = 0, 1, 2
VATTN_KV_DEVICE, VATTN_KV_HOST = 0, 1
VATTN_GUARANTEE_DENOMINATOR, VATTN_GUARANTEE_OUTPUT = 0, 1
VATTN_OK, VATTN_EINVAL, VATTN_ENOMEM, VATTN_ECUDA, VATTN_ESCRATCH = 0, -1, -2, -3, -4
VATTN_DEV_BAD_SEQLEN, VATTN_DEV_BAD_PAGE, VATTN_DEV_TIMEOUT = 1, 2, 4

# every symbol include/vattn.h declares
EXPORTS = ("vattn_create", "vattn_decode", "vattn_dense_decode", "vattn_dense_decode_static",
           "vattn_last_error", "vattn_check_bounded_wait",
           "vattn_workspace_bytes", "vattn_set_timing", "vattn_score_pass_ms",
           "vattn_last_launch_count", "vattn_strerror", "vattn_destroy")


class vattn_config(C.Structure):
    _fields_ = [("num_q_heads", C.c_int), ("num_kv_heads", C.c_int), ("head_dim", C.c_int),
                ("dtype", C.c_int), ("page_size", C.c_int), ("max_batch", C.c_int),
                ("max_ctx", C.c_int), ("proxy", C.c_int), ("proxy_rank", C.c_int),
                ("kv_location", C.c_int)]


class vattn_params(C.Structure):
    _fields_ = [("sinks", C.c_int), ("window", C.c_int),
                ("topk_abs", C.c_int), ("topk_num", C.c_int), ("topk_den", C.c_int),
                ("pilot_min", C.c_int), ("pilot_num", C.c_int), ("pilot_den", C.c_int),
                ("eps", C.c_float), ("delta", C.c_float), ("seed", C.c_uint64),
                ("num_pages", C.c_int),
                ("k_t_cache", C.c_void_p), ("k_proj_cache", C.c_void_p), ("proj_basis", C.c_void_p),
                ("guarantee", C.c_int), ("topp_num", C.c_int), ("topp_den", C.c_int),
                ("batch_offset", C.c_int), ("head_offset", C.c_int)]


class VattnError(RuntimeError):
    pass


_LIB = None


def lib():
    """The loaded libvattn.so (raises if it was not built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m verified_sparse_attention_b200.csrc.build`")
        L = C.CDLL(LIB_PATH)
        P, I = C.c_void_p, C.c_int
        L.vattn_create.argtypes = [C.POINTER(C.c_void_p), C.POINTER(vattn_config)]
        L.vattn_create.restype = I
        L.vattn_decode.argtypes = [P, P, P, P, P, P, I, C.POINTER(vattn_params), P, P, P, P, P, P]
        L.vattn_decode.restype = I
        L.vattn_dense_decode.argtypes = [P, P, P, P, P, P, I, I, P, P]
        L.vattn_dense_decode.restype = I
        L.vattn_dense_decode_static.argtypes = [C.POINTER(vattn_config), P, P, P, P, P, I, I, P, P]
        L.vattn_dense_decode_static.restype = I
        L.vattn_check_bounded_wait.argtypes = [P, I, P]
        L.vattn_check_bounded_wait.restype = I
        L.vattn_last_error.argtypes = [P, I]
        L.vattn_last_error.restype = I
        L.vattn_workspace_bytes.argtypes = [P]
        L.vattn_workspace_bytes.restype = C.c_size_t
        L.vattn_set_timing.argtypes = [P, I]
        L.vattn_set_timing.restype = I
        L.vattn_score_pass_ms.argtypes = [P, C.POINTER(C.c_double), C.POINTER(C.c_int), I]
        L.vattn_score_pass_ms.restype = I
        L.vattn_last_launch_count.argtypes = [P]
        L.vattn_last_launch_count.restype = I
        L.vattn_strerror.argtypes = [I]
        L.vattn_strerror.restype = C.c_char_p
        L.vattn_destroy.argtypes = [P]
        L.vattn_destroy.restype = None
        _LIB = L
    return _LIB


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _check(rc, what):
    if rc != VATTN_OK:
        raise VattnError(f"{what}: {lib().vattn_strerror(rc).decode()} ({rc})")
    return rc


def _stream_ptr(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def vattn_create(config):
    """Create a context from a vattn_config (or a dict of its fields); returns the handle."""
    if isinstance(config, dict):
        config = vattn_config(**config)
    h = C.c_void_p()
    _check(lib().vattn_create(C.byref(h), C.byref(config)), "vattn_create")
    return h.value


def vattn_decode(ctx, q, k_cache, v_cache, page_table, seq_lens, batch, params, out, sel_idx,
                 sel_count, budgets, head_need, stream=None, check=True):
    """One sparse decode step (see include/vattn.h); returns the C return code."""
    if isinstance(params, dict):
        params = vattn_params(**params)
    rc = lib().vattn_decode(ctx, _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(page_table),
                            _ptr(seq_lens), int(batch), C.byref(params), _ptr(out), _ptr(sel_idx),
                            _ptr(sel_count), _ptr(budgets), _ptr(head_need), _stream_ptr(stream))
    return _check(rc, "vattn_decode") if check else rc


def vattn_dense_decode(ctx, q, k_cache, v_cache, page_table, seq_lens, batch, num_pages, out,
                       stream=None, check=True):
    rc = lib().vattn_dense_decode(ctx, _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(page_table),
                                  _ptr(seq_lens), int(batch), int(num_pages), _ptr(out),
                                  _stream_ptr(stream))
    return _check(rc, "vattn_dense_decode") if check else rc


def vattn_dense_decode_static(config, q, k_cache, v_cache, page_table, seq_lens, batch, num_pages,
                              out, stream=None, check=True):
    """Dense decode without a context or any allocation (scratch: a fixed
    device array in the library, shared by every call on a device)."""
    if isinstance(config, dict):
        config = vattn_config(**config)
    rc = lib().vattn_dense_decode_static(C.byref(config), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                         _ptr(page_table), _ptr(seq_lens), int(batch),
                                         int(num_pages), _ptr(out), _stream_ptr(stream))
    return _check(rc, "vattn_dense_decode_static") if check else rc


def vattn_last_error(ctx, sync=True):
    return lib().vattn_last_error(ctx, 1 if sync else 0)


def vattn_check_bounded_wait(ctx, tries, stream=None, check=True):
    """Run the device wait self-check (sets VATTN_DEV_TIMEOUT in the error word)."""
    rc = lib().vattn_check_bounded_wait(ctx, int(tries), _stream_ptr(stream))
    return _check(rc, "vattn_check_bounded_wait") if check else rc


def vattn_workspace_bytes(ctx):
    return lib().vattn_workspace_bytes(ctx)


def vattn_set_timing(ctx, period):
    """Time the score pass of every `period`-th decode call (True = every call, 0 / False = off)."""
    return _check(lib().vattn_set_timing(ctx, int(period)), "vattn_set_timing")


def vattn_score_pass_ms(ctx, reset=True):
    """(total milliseconds, number of timed score passes) since the last reset."""
    ms, n = C.c_double(), C.c_int()
    _check(lib().vattn_score_pass_ms(ctx, C.byref(ms), C.byref(n), 1 if reset else 0),
           "vattn_score_pass_ms")
    return ms.value, n.value


def vattn_last_launch_count(ctx):
    return lib().vattn_last_launch_count(ctx)


def vattn_strerror(code):
    return lib().vattn_strerror(code).decode()


def vattn_destroy(ctx):
    if ctx:
        lib().vattn_destroy(ctx)
