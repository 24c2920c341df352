"""ctypes view of libqsa.so: the C ABI declared in include/qsa.h."""
from __future__ import annotations

import ctypes
import os

from .build import LIB_PATH

c_int32, c_int64, c_size_t, c_void_p, c_float = (ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t,
                                                 ctypes.c_void_p, ctypes.c_float)

QSA_OK = 0
QSA_F32, QSA_BF16, QSA_FP8_E4M3 = 0, 1, 2


class QsaCacheStruct(ctypes.Structure):
    """Mirror of `qsa_cache` in include/qsa.h."""
    _fields_ = [
        ("num_pages", c_int32), ("page_size", c_int32), ("num_kv_heads", c_int32),
        ("head_dim", c_int32), ("idx_dim", c_int32), ("kv_dtype", c_int32),
        ("k_cache", c_void_p), ("v_cache", c_void_p), ("k_scale", c_void_p),
        ("v_scale", c_void_p), ("kc", c_void_p), ("ring", c_void_p), ("ring_rows", c_int32),
        ("block_table", c_void_p), ("max_pages_per_req", c_int32),
    ]


# name -> (restype, argtypes); exactly the entry points of include/qsa.h
SIGNATURES = {
    "qsa_status_string": (ctypes.c_char_p, [c_int32]),
    "qsa_abi_version": (c_int32, []),
    "qsa_kc_page_bytes": (c_size_t, [c_int32, c_int32]),
    "qsa_compress_append": (c_int32, [ctypes.POINTER(QsaCacheStruct), c_int32, c_void_p, c_void_p,
                                      c_void_p, c_int32, c_void_p]),
    "qsa_index_topk_workspace_bytes": (c_size_t, [c_int32, c_int32]),
    "qsa_index_topk": (c_int32, [ctypes.POINTER(QsaCacheStruct), c_int32, c_void_p, c_void_p,
                                 c_void_p, c_int32, c_int32, c_void_p, c_void_p, c_void_p,
                                 c_size_t, c_void_p]),
    "qsa_sparse_decode_workspace_bytes": (c_size_t, [c_int32] * 7),
    "qsa_sparse_decode": (c_int32, [ctypes.POINTER(QsaCacheStruct), c_int32, c_int32, c_int32,
                                    c_void_p, c_int32, c_void_p, c_void_p, c_int32, c_float,
                                    c_int32, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "qsa_sparse_decode_merged": (c_int32, [ctypes.POINTER(QsaCacheStruct), c_int32, c_int32, c_int32,
                                           c_void_p, c_int32, c_void_p, c_void_p, c_int32, c_float,
                                           c_int32, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                           c_size_t, c_void_p]),
    "qsa_sparse_decode_splits": (c_int32, [ctypes.POINTER(QsaCacheStruct), c_int32, c_int32, c_int32,
                                           c_void_p, c_int32, c_void_p, c_void_p, c_int32, c_float,
                                           c_int32, c_int32, c_int32, c_void_p, c_void_p, c_void_p,
                                           c_size_t, c_void_p]),
    "qsa_lse_merge": (c_int32, [c_int32, c_int64, c_int32, c_void_p, c_void_p, c_void_p, c_void_p,
                                c_void_p]),
    "qsa_index_topk_noalloc": (c_int32, [ctypes.POINTER(QsaCacheStruct), c_int32, c_void_p,
                                         c_void_p, c_void_p, c_int32, c_int32, c_void_p,
                                         c_void_p]),
    "qsa_index_topk_tokens": (c_int32, [ctypes.POINTER(QsaCacheStruct), c_int32, c_void_p,
                                        c_void_p, c_void_p, c_int32, c_int32, c_int32, c_void_p,
                                        c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "qsa_kcn_page_bytes": (c_size_t, [c_int32, c_int32]),
    "qsa_compress_append_norm": (c_int32, [ctypes.POINTER(QsaCacheStruct), c_void_p, c_void_p,
                                           c_void_p, c_float, c_int32, c_void_p, c_void_p,
                                           c_void_p, c_int32, c_void_p]),
    "qsa_index_topk_norm": (c_int32, [ctypes.POINTER(QsaCacheStruct), c_void_p, c_int32, c_void_p,
                                      c_void_p, c_void_p, c_int32, c_int32, c_void_p, c_void_p,
                                      c_void_p, c_size_t, c_void_p]),
    "qsa_sparse_prefill_workspace_bytes": (c_size_t, [c_int32] * 6),
    "qsa_sparse_prefill": (c_int32, [ctypes.POINTER(QsaCacheStruct), c_int32, c_int32, c_int32,
                                     c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int32,
                                     c_int32, c_int32, c_int32, c_float, c_void_p, c_void_p,
                                     c_void_p, c_void_p, c_size_t, c_void_p]),
    "qsa_get_device_error": (c_int32, [c_void_p, ctypes.POINTER(ctypes.c_uint32)]),
    "qsa_session_create": (c_int32, [ctypes.POINTER(QsaCacheStruct), c_int32, c_int32, c_int32,
                                     c_int32, c_int32, c_int32, c_int32, c_int32, c_float,
                                     c_void_p, ctypes.POINTER(c_void_p)]),
    "qsa_session_step_host": (c_int32, [c_void_p] * 10),
    "qsa_session_streams": (c_int32, [c_void_p, ctypes.POINTER(c_void_p), ctypes.POINTER(c_void_p),
                                      ctypes.POINTER(c_void_p)]),
    "qsa_session_synchronize": (c_int32, [c_void_p]),
    "qsa_session_destroy": (c_int32, [c_void_p]),
}

_lib = None


def load() -> ctypes.CDLL:
    """Loads libqsa.so; raises if it has not been built (there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libqsa.so not found at {LIB_PATH}; build it with "
                "`python -m sparse_attention_decode_compress_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib
