"""ctypes declarations of the C-ABI in include/pariskv.h (libpariskv.so).

Loading fails loudly when the in-tree library is missing: there is no CPU or
PyTorch fallback for any step of the path.
"""
from __future__ import annotations

import ctypes as C
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpariskv.so")

# every symbol include/pariskv.h declares
EXPORTS = (
    "pk_default_params", "pk_build_index", "pk_append", "pk_search", "pk_search_debug",
    "pk_attend", "pk_free", "pk_status_str", "pk_last_device_error", "pk_get_info",
    "pk_export_index", "pk_magnitude_levels", "pk_resolve", "pk_trace_enable", "pk_trace_read",
    "pk_select_candidates_noalloc", "pk_attend_dense", "pk_search_heads", "pk_attend_heads",
    "pk_append_stage", "pk_append_publish",
)

PK_OK, PK_ERR_INVALID_ARG, PK_ERR_CAPACITY, PK_ERR_OOM, PK_ERR_CUDA, PK_ERR_TIMEOUT, \
    PK_ERR_DEVICE_CHECK, PK_ERR_UNSUPPORTED = range(8)
PK_F32, PK_BF16 = 0, 1
PK_KV_DEVICE, PK_KV_HOST_PINNED = 0, 1
KERNELS = ("encode", "query_prep", "collision_scan", "compact", "rerank_topk", "topk_merge",
           "gather_attend")


class pk_params(C.Structure):
    _fields_ = [
        ("batch", C.c_int32), ("n_kv_heads", C.c_int32), ("group", C.c_int32),
        ("head_dim", C.c_int32), ("sub_dim", C.c_int32), ("topk", C.c_int32),
        ("n_cap", C.c_int64), ("cand_budget", C.c_int64), ("collision_ratio", C.c_float),
        ("attn_scale", C.c_float), ("rot_seed", C.c_uint64), ("kv_dtype", C.c_int32),
        ("kv_location", C.c_int32),
    ]


class pk_info(C.Structure):
    _fields_ = [
        ("n", C.c_int64), ("n_cap", C.c_int64), ("bh", C.c_int32), ("nchunks", C.c_int32),
        ("chunk", C.c_int64), ("cand", C.c_int64), ("coll", C.c_int64),
        ("index_bytes", C.c_int64), ("kv_bytes", C.c_int64), ("kv_location", C.c_int32),
        ("num_sms", C.c_int32), ("n_staged", C.c_int64),
    ]


class pk_debug_out(C.Structure):
    _fields_ = [
        ("qt", C.c_void_p), ("qnorm", C.c_void_p), ("bonus", C.c_void_p), ("S", C.c_void_p),
        ("hist", C.c_void_p), ("sstar", C.c_void_p), ("cand", C.c_void_p), ("cand_est", C.c_void_p),
    ]


def load() -> C.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            "libpariskv.so is not built (%s); build it with `python -m kv_cache_top_b200.build`"
            % LIB_PATH)
    lib = C.CDLL(LIB_PATH)
    P, I32, I64, F32 = C.c_void_p, C.c_int32, C.c_int64, C.c_float
    st = C.c_int
    lib.pk_default_params.restype = None
    lib.pk_default_params.argtypes = [C.POINTER(pk_params)]
    lib.pk_build_index.restype = st
    lib.pk_build_index.argtypes = [P, P, I64, C.POINTER(pk_params), P, C.POINTER(P)]
    lib.pk_append.restype = st
    lib.pk_append.argtypes = [P, P, P, I64, P]
    lib.pk_append_stage.restype = st
    lib.pk_append_stage.argtypes = [P, P, P, I64, I64, P]
    lib.pk_append_publish.restype = st
    lib.pk_append_publish.argtypes = [P, P]
    lib.pk_search.restype = st
    lib.pk_search.argtypes = [P, P, I32, P, P, P]
    lib.pk_search_debug.restype = st
    lib.pk_search_debug.argtypes = [P, P, I32, P, P, C.POINTER(pk_debug_out), P]
    lib.pk_attend.restype = st
    lib.pk_attend.argtypes = [P, P, P, I32, P, P]
    lib.pk_search_heads.restype = st
    lib.pk_search_heads.argtypes = [P, P, I32, P, P, P]
    lib.pk_attend_heads.restype = st
    lib.pk_attend_heads.argtypes = [P, P, P, I32, P, P]
    lib.pk_attend_dense.restype = st
    lib.pk_attend_dense.argtypes = [P, P, P, I32, P, P, I64, I32, P, P]
    lib.pk_free.restype = None
    lib.pk_free.argtypes = [P]
    lib.pk_status_str.restype = C.c_char_p
    lib.pk_status_str.argtypes = [st]
    lib.pk_last_device_error.restype = st
    lib.pk_last_device_error.argtypes = [P, C.POINTER(I64)]
    lib.pk_get_info.restype = st
    lib.pk_get_info.argtypes = [P, C.POINTER(pk_info)]
    lib.pk_export_index.restype = st
    lib.pk_export_index.argtypes = [P, P, P, P, P]
    lib.pk_magnitude_levels.restype = st
    lib.pk_magnitude_levels.argtypes = [I32, I32, P, P]
    lib.pk_resolve.restype = st
    lib.pk_resolve.argtypes = [I64, I64, F32, I32, C.POINTER(I64), C.POINTER(I64)]
    lib.pk_trace_enable.restype = st
    lib.pk_trace_enable.argtypes = [P, I32]
    lib.pk_trace_read.restype = st
    lib.pk_trace_read.argtypes = [P, P, P]
    lib.pk_select_candidates_noalloc.restype = st
    lib.pk_select_candidates_noalloc.argtypes = [P, I64, I64, P, P]
    return lib
