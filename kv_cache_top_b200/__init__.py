"""B200 (sm_100a) ParisKV decode-time KV-cache retrieval.

A thin binding over ``libpariskv.so`` (C-ABI in ``include/pariskv.h``): the
functions below have the C names and only marshal arguments (tensor data
pointers, the current CUDA stream).  Every step of the path runs in the
library's CUDA kernels; PyTorch supplies device memory and streams.
"""
from __future__ import annotations

import ctypes as C

import numpy as np

from . import _lib
from ._lib import (KERNELS, PK_BF16, PK_F32, PK_KV_DEVICE, PK_KV_HOST_PINNED, PK_OK, pk_debug_out,
                   pk_info, pk_params)

_handle = None


def _L():
    """The loaded library: loaded on first use, so that importing the package
    (e.g. to build it) does not need it; every API call fails loudly (an
    ImportError) when it is missing."""
    global _handle
    if _handle is None:
        _handle = _lib.load()
    return _handle


def __getattr__(name):
    if name == "lib":
        return _L()
    raise AttributeError("module %r has no attribute %r" % (__name__, name))

__all__ = [
    "PkError", "pk_default_params", "pk_build_index", "pk_append", "pk_search", "pk_search_debug",
    "pk_attend", "pk_free", "pk_status_str", "pk_last_device_error", "pk_get_info",
    "pk_export_index", "pk_magnitude_levels", "pk_resolve", "pk_trace_enable", "pk_trace_read",
    "pk_select_candidates_noalloc", "pk_attend_dense", "pk_search_heads", "pk_attend_heads",
    "pk_append_stage", "pk_append_publish", "pk_params", "pk_info", "pk_debug_out", "PK_F32",
    "PK_BF16", "PK_KV_DEVICE", "PK_KV_HOST_PINNED", "KERNELS", "lib",
]


class PkError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (what, pk_status_str(status), status))


def _check(status: int, what: str):
    if status != PK_OK:
        raise PkError(status, what)


def _ptr(x):
    """Data pointer of a tensor (or an int address, or None)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def pk_status_str(status: int) -> str:
    return _L().pk_status_str(status).decode()


def pk_default_params(**kw) -> pk_params:
    p = pk_params()
    _L().pk_default_params(C.byref(p))
    for k, v in kw.items():
        if not hasattr(p, k):
            raise AttributeError("pk_params has no field %r" % k)
        setattr(p, k, v)
    return p


def pk_build_index(K, V, n: int, params: pk_params, stream=None) -> C.c_void_p:
    h = C.c_void_p()
    _check(_L().pk_build_index(_ptr(K), _ptr(V), int(n), C.byref(params), _stream(stream), C.byref(h)),
           "pk_build_index")
    return h


def pk_append(index, k_new, v_new, n_new: int, stream=None):
    _check(_L().pk_append(index, _ptr(k_new), _ptr(v_new), int(n_new), _stream(stream)), "pk_append")


def pk_append_stage(index, k_new, v_new, n_new: int, src_stride: int = 0, stream=None):
    """Encode n_new rows per pair of k_new/v_new ([BH][src_stride][D]) into the
    index without making them visible to search (see pk_append_publish)."""
    _check(_L().pk_append_stage(index, _ptr(k_new), _ptr(v_new), int(n_new), int(src_stride), _stream(stream)),
           "pk_append_stage")


def pk_append_publish(index, stream=None):
    """Make the staged keys visible to work enqueued on `stream` after this call."""
    _check(_L().pk_append_publish(index, _stream(stream)), "pk_append_publish")


def pk_search(index, q, topk: int, out_idx, out_score=None, stream=None):
    _check(_L().pk_search(index, _ptr(q), int(topk), _ptr(out_idx), _ptr(out_score), _stream(stream)),
           "pk_search")


def pk_search_debug(index, q, topk: int, out_idx, out_score=None, dbg: dict | None = None,
                    stream=None):
    d = pk_debug_out()
    for k, v in (dbg or {}).items():
        setattr(d, k, _ptr(v))
    _check(_L().pk_search_debug(index, _ptr(q), int(topk), _ptr(out_idx), _ptr(out_score), C.byref(d),
                               _stream(stream)), "pk_search_debug")


def pk_attend(index, q, sel_idx, topk: int, out, stream=None):
    _check(_L().pk_attend(index, _ptr(q), _ptr(sel_idx), int(topk), _ptr(out), _stream(stream)),
           "pk_attend")


def pk_attend_dense(index, q, sel_idx, topk: int, dense_K, dense_V, dense_len: int, out, stream=None):
    """Attention over the selected rows and the dense (sink + local) rows of
    dense_K/dense_V [BH][stride][D] under one softmax."""
    dstride = dense_K.shape[-2] if dense_K is not None and hasattr(dense_K, "shape") else 0
    _check(_L().pk_attend_dense(index, _ptr(q), _ptr(sel_idx), int(topk), _ptr(dense_K), _ptr(dense_V),
                                int(dstride), int(dense_len), _ptr(out), _stream(stream)), "pk_attend_dense")


def pk_search_heads(index, q, topk: int, out_idx, out_score=None, stream=None):
    """Per-query-head retrieval: out_idx [batch][H*G][topk]."""
    _check(_L().pk_search_heads(index, _ptr(q), int(topk), _ptr(out_idx), _ptr(out_score), _stream(stream)),
           "pk_search_heads")


def pk_attend_heads(index, q, sel_idx, topk: int, out, stream=None):
    """Attention of every query head over its own rows sel_idx [batch][H*G][topk]."""
    _check(_L().pk_attend_heads(index, _ptr(q), _ptr(sel_idx), int(topk), _ptr(out), _stream(stream)),
           "pk_attend_heads")


def pk_free(index):
    _L().pk_free(index)


def pk_last_device_error(index):
    """(status, detail): waits for the device, then reads and clears the
    index's device-check word."""
    det = C.c_int64(0)
    st = _L().pk_last_device_error(index, C.byref(det))
    return st, det.value


def pk_get_info(index) -> pk_info:
    info = pk_info()
    _check(_L().pk_get_info(index, C.byref(info)), "pk_get_info")
    return info


def pk_export_index(index, codes=None, records=None, occ=None, stream=None):
    _check(_L().pk_export_index(index, _ptr(codes), _ptr(records), _ptr(occ), _stream(stream)),
           "pk_export_index")


def pk_magnitude_levels(m: int = 8, L: int = 8):
    lev = np.empty(L, np.float32)
    thr = np.empty(L - 1, np.float32)
    _check(_L().pk_magnitude_levels(m, L, lev.ctypes.data, thr.ctypes.data), "pk_magnitude_levels")
    return lev, thr


def pk_resolve(n: int, cand_budget: int = 0, collision_ratio: float = 0.0, topk: int = 100):
    c = C.c_int64()
    r = C.c_int64()
    _check(_L().pk_resolve(n, cand_budget, collision_ratio, topk, C.byref(c), C.byref(r)), "pk_resolve")
    return c.value, r.value


def pk_trace_enable(index, on: bool = True):
    _check(_L().pk_trace_enable(index, 1 if on else 0), "pk_trace_enable")


def pk_trace_read(index):
    """{kernel: (launches, total_ms)} since the last read (synchronises)."""
    n = np.zeros(len(KERNELS), np.int64)
    ms = np.zeros(len(KERNELS), np.float64)
    _check(_L().pk_trace_read(index, n.ctypes.data, ms.ctypes.data), "pk_trace_read")
    return {k: (int(n[i]), float(ms[i])) for i, k in enumerate(KERNELS)}


def pk_select_candidates_noalloc(S, n: int, C: int, cand, stream=None):
    """Top-C candidate ids of one score row with no device allocation (see
    include/pariskv.h): for callers that cannot allocate at that moment."""
    _check(_L().pk_select_candidates_noalloc(_ptr(S), int(n), int(C), _ptr(cand), _stream(stream)),
           "pk_select_candidates_noalloc")
