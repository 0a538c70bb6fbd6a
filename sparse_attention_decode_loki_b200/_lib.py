"""ctypes loader and prototypes for libloki.so (the C ABI in include/loki.h).

The shared library is required: importing this module without it raises
ImportError. There is no Python or CPU fallback for any entry point.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libloki.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python sparse_attention_decode_loki_b200/build.py`"
    )

lib = ctypes.CDLL(LIB_PATH)

c_int, c_int64, c_size_t, c_float = ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
c_void_p, c_char_p = ctypes.c_void_p, ctypes.c_char_p

# name -> (restype, argtypes), in the order of include/loki.h
PROTOTYPES = {
    "loki_status_string": (c_char_p, [c_int]),
    "loki_last_error": (c_char_p, []),
    "loki_device_error": (c_int, [ctypes.POINTER(c_int), c_int]),
    "loki_calibrate_workspace_size": (c_size_t, [c_int64, c_int, c_int]),
    "loki_calibrate_pca": (c_int, [c_void_p, c_int, c_int64, c_int, c_int, c_void_p, c_void_p,
                                   c_void_p, c_size_t, c_void_p]),
    "loki_append_keys": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int,
                                 c_int, c_int, c_int64, c_int64, c_int, c_void_p]),
    "loki_append_keys_plane": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_int, c_int, c_int, c_int, c_int, c_int64, c_int64, c_int,
                                       c_void_p]),
    "loki_decode_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int64, c_int, c_int, c_int64]),
    "loki_decode_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
                                      c_int64, c_int64, c_int, c_int, c_int64, c_float, c_int,
                                      c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "loki_decode_attention_plane": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                                            c_void_p, c_int, c_int, c_int, c_int64, c_int64, c_int,
                                            c_int, c_int64, c_float, c_int, c_void_p, c_void_p,
                                            c_void_p, c_size_t, c_void_p]),
    "loki_decode_step": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                 c_void_p, c_int, c_int, c_int, c_int, c_int, c_int64, c_int64,
                                 c_int, c_int, c_int64, c_float, c_int, c_void_p, c_void_p,
                                 c_void_p, c_size_t, c_void_p]),
    "loki_decode_attention_fused": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                                            c_void_p, c_int, c_int, c_int, c_int64, c_int64, c_int,
                                            c_int, c_int64, c_float, c_int, c_void_p, c_void_p,
                                            c_void_p]),
    "loki_decode_attention_noalloc": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int,
                                              c_int, c_int64, c_int64, c_int, c_int, c_int64,
                                              c_float, c_int, c_void_p, c_void_p, c_void_p]),
    "loki_paged_decode_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int, c_int, c_int,
                                                    c_int, c_int64]),
    "loki_decode_attention_paged": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                                            c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
                                            c_int, c_int, c_int64, c_int, c_int, c_int64, c_float,
                                            c_int, c_void_p, c_void_p, c_void_p, c_size_t,
                                            c_void_p]),
    "loki_append_keys_paged": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_int, c_void_p, c_void_p, c_int, c_int, c_int, c_int,
                                       c_int, c_int64, c_int, c_int, c_void_p]),
    "loki_project_query": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_void_p,
                                   c_void_p]),
    "loki_score_lowdim": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int64, c_int64, c_int,
                                  c_int, c_int, c_void_p, c_void_p]),
    "loki_topk_workspace_size": (c_size_t, [c_int64, c_int64, c_int64]),
    "loki_topk": (c_int, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p, c_size_t,
                          c_void_p]),
    "loki_sparse_attention_workspace_size": (c_size_t, [c_int, c_int, c_int64, c_int]),
    "loki_sparse_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
                                      c_int64, c_int64, c_int, c_int64, c_float, c_int, c_void_p,
                                      c_void_p, c_size_t, c_void_p]),
    "loki_pca_attention_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int64, c_int]),
    "loki_pca_attention": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_int, c_int,
                                   c_int, c_int64, c_int64, c_int, c_int, c_float, c_int,
                                   c_void_p, c_void_p, c_size_t, c_void_p]),
    "loki_decode_prerotary_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int64, c_int, c_int,
                                                        c_int64]),
    "loki_decode_attention_prerotary": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                                c_int, c_void_p, c_int, c_int, c_int, c_int64,
                                                c_int64, c_int, c_int, c_int64, c_float, c_int,
                                                c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "loki_append_keys_prerotary": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                           c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int,
                                           c_int64, c_int64, c_int, c_void_p]),
    "dense_decode_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int64, c_int]),
    "dense_decode_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int64,
                                       c_int64, c_int, c_float, c_int, c_void_p, c_void_p, c_size_t,
                                       c_void_p]),
}

for _name, (_res, _args) in PROTOTYPES.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args

STATUS = {0: "LOKI_OK", 1: "LOKI_ERR_INVALID_ARG", 2: "LOKI_ERR_UNSUPPORTED",
          3: "LOKI_ERR_WORKSPACE_TOO_SMALL", 4: "LOKI_ERR_CUDA"}
DTYPE_F32 = 0
DTYPE_BF16 = 1


class LokiError(RuntimeError):
    """A non-OK status from the C library; `.status` holds the code."""

    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.loki_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS.get(status, status)}: {msg}")


def check(status: int, where: str) -> None:
    if status != 0:
        raise LokiError(status, where)
