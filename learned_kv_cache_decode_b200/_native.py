"""ctypes declarations for libdms.so (the C ABI in include/dms.h).

The shared library is built in-tree by ``learned_kv_cache_decode_b200.build``.
If it is missing, importing this module raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# DMS_LIBRARY=debug selects the build with device-side bounds checks
# (libdms_debug.so); the default is libdms.so.
LIB_PATH = os.path.join(_HERE, "libdms_debug.so" if os.environ.get("DMS_LIBRARY") == "debug" else "libdms.so")

DMS_OK = 0
DMS_ERR_INVALID = 1
DMS_ERR_POOL_EXHAUSTED = 2
DMS_ERR_CUDA = 3
DMS_ERR_TIMEOUT = 4
DMS_ERR_POISONED = 5
DMS_ERR_STREAM_FULL = 6
DMS_ERR_BAD_SEQ = 7

DMS_BF16 = 0
DMS_F32 = 1

DMS_ATTN_AUTO = 0
DMS_ATTN_SIMT = 1
DMS_ATTN_MMA = 2

EXPORTS = ("dms_cache_create", "dms_cache_destroy", "dms_cache_reset", "dms_seq_reset", "dms_append",
           "dms_decode_attention", "dms_stats", "dms_snapshot", "dms_gather_kv", "dms_get_status",
           "dms_status_string", "dms_launch_count", "dms_decode_attention_noalloc", "dms_decode_step",
           "dms_append_keyed", "dms_decode_step_keyed", "dms_selftest_bounded_waits",
           "dms_decode_step_qkeyed", "dms_alpha_from_logit", "dms_stats_host")

DMS_NOALLOC_MAX_STREAMS = 512
DMS_NOALLOC_MAX_PIECES = 1024


class DmsConfig(ctypes.Structure):
    _fields_ = [
        ("max_seqs", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("max_pages", ctypes.c_int32),
        ("max_pages_per_stream", ctypes.c_int32),
        ("dtype", ctypes.c_int),
        ("attn_kernel", ctypes.c_int),
    ]


class DmsPagedKv(ctypes.Structure):
    """Caller-owned paged K/V for dms_decode_attention_noalloc."""
    _fields_ = [
        ("kv_pool", ctypes.c_void_p),
        ("page_table", ctypes.c_void_p),
        ("retained", ctypes.c_void_p),
        ("max_seqs", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("max_pages", ctypes.c_int32),
        ("max_pages_per_stream", ctypes.c_int32),
        ("dtype", ctypes.c_int),
    ]


class DmsError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


_lib = None


def load() -> ctypes.CDLL:
    """Load libdms.so, declaring every entry point. Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m learned_kv_cache_decode_b200.build` "
            "(nvcc, sm_100a). There is no CPU fallback.")
    L = ctypes.CDLL(LIB_PATH)
    p, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    st = ctypes.c_int
    L.dms_cache_create.argtypes = [ctypes.POINTER(DmsConfig), ctypes.POINTER(p)]
    L.dms_cache_create.restype = st
    L.dms_cache_destroy.argtypes = [p]
    L.dms_cache_destroy.restype = st
    L.dms_cache_reset.argtypes = [p, p]
    L.dms_cache_reset.restype = st
    L.dms_seq_reset.argtypes = [p, p, i32]
    L.dms_seq_reset.restype = st
    L.dms_append.argtypes = [p, p, i32, p, p, i32, p, p, p]
    L.dms_append.restype = st
    L.dms_decode_attention.argtypes = [p, p, i32, p, p, i32, ctypes.c_float, p, ctypes.c_int]
    L.dms_decode_attention.restype = st
    L.dms_stats.argtypes = [p, p, p, p, p, p]
    L.dms_stats.restype = st
    L.dms_stats_host.argtypes = [p, p, p, p, ctypes.POINTER(ctypes.c_double)]
    L.dms_stats_host.restype = st
    L.dms_snapshot.argtypes = [p, p, p, p, p, p, p, p, p]
    L.dms_snapshot.restype = st
    L.dms_gather_kv.argtypes = [p, p, i32, i32, i32, p, p]
    L.dms_gather_kv.restype = st
    L.dms_get_status.argtypes = [p, p]
    L.dms_get_status.restype = st
    L.dms_selftest_bounded_waits.argtypes = [p, p, p]
    L.dms_selftest_bounded_waits.restype = st
    L.dms_status_string.argtypes = [st]
    L.dms_status_string.restype = ctypes.c_char_p
    L.dms_launch_count.argtypes = [p]
    L.dms_launch_count.restype = i64
    L.dms_decode_step.argtypes = [p, p, i32, p, p, p, p, p, i32, ctypes.c_float, p, ctypes.c_int]
    L.dms_decode_step.restype = st
    L.dms_append_keyed.argtypes = [p, p, i32, p, p, i32, p, p, i32]
    L.dms_append_keyed.restype = st
    L.dms_decode_step_keyed.argtypes = [p, p, i32, p, p, p, i32, p, i32, ctypes.c_float, p, ctypes.c_int]
    L.dms_decode_step_keyed.restype = st
    L.dms_decode_step_qkeyed.argtypes = [p, p, i32, p, p, p, p, i32, i32, i32, ctypes.c_float, p, ctypes.c_int]
    L.dms_decode_step_qkeyed.restype = st
    L.dms_alpha_from_logit.argtypes = [p, p, ctypes.c_int, i32, i32, i32, i32, i32, i32, p]
    L.dms_alpha_from_logit.restype = st
    L.dms_decode_attention_noalloc.argtypes = [p, ctypes.POINTER(DmsPagedKv), i32, p, p, i32, ctypes.c_float, p,
                                               ctypes.c_int]
    L.dms_decode_attention_noalloc.restype = st
    _lib = L
    return L


def status_string(code: int) -> str:
    try:
        return load().dms_status_string(code).decode()
    except ImportError:
        return f"status {code}"


def check(code: int, where: str) -> None:
    if code != DMS_OK:
        raise DmsError(code, where)
