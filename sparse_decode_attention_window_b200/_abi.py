"""ctypes binding of libkvc.so: the C ABI of include/kvc.h, one Python function
per entry point, same names. Argument marshalling only - device pointers come
from torch tensors, the stream from torch's current CUDA stream; every step of
the hot path runs in the library's kernels. Loading fails loudly if the library
is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkvc.so")

KVC_OK, KVC_ERR_INVALID_ARG, KVC_ERR_SHAPE, KVC_ERR_UNSUPPORTED = 0, 1, 2, 3
KVC_ERR_CAPACITY, KVC_ERR_CUDA, KVC_ERR_WORKSPACE, KVC_ERR_DEVICE = 4, 5, 6, 7
KVC_BF16, KVC_FP32 = 0, 1
KVC_POL_TOPB, KVC_POL_MASS_COUNT, KVC_POL_LOCAL, KVC_POL_SPECIAL, KVC_POL_FULL, KVC_POL_CHUNK = 0, 1, 2, 3, 4, 5
KVC_WS_SCORE, KVC_WS_SELECT, KVC_WS_DECODE = 0, 1, 2

# every symbol the header declares
EXPORTS = ["kvc_score", "kvc_select", "kvc_alloc_budgets", "kvc_layout", "kvc_compact", "kvc_layout_compact",
           "kvc_append",
           "kvc_append_window",
           "kvc_decode_attn", "kvc_workspace_size", "kvc_get_status", "kvc_last_error", "kvc_version",
           "kvc_launch_count", "kvc_decode_attn_noalloc", "kvc_append_decode", "kvc_append_decode_chain", "kvc_select_chunks",
           "kvc_retained_mass", "kvc_profile_heads", "kvc_check_wait_limit", "kvc_diag_set_path",
           "kvc_diag_get_path"]

# kvc_diag_set_path knobs and choices (cross-checks only)
KVC_DIAG = {
    "score": (0, {"auto": 0, "twopass": 1, "simt": 2, "cluster": 3}),
    "select": (1, {"auto": 0, "cta": 1}),
    "compact": (2, {"auto": 0, "grid": 1}),
    "decode": (3, {"auto": 0, "simt": 1, "tc": 2}),
    "decode_split": (4, {"auto": 0, "tokens": 1}),
    "score_k": (5, {"auto": 0, **{str(k): k for k in range(1, 17)}}),
}


class KvcShape(ctypes.Structure):
    _fields_ = [("n_slots", ctypes.c_int32), ("G", ctypes.c_int32), ("d", ctypes.c_int32), ("L", ctypes.c_int32),
                ("w", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("batch", ctypes.c_int32),
                ("dtype", ctypes.c_int32)]


class KvcError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn} failed with status {status}: {msg}")
        self.status = status


_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load libkvc.so (raises OSError if it is missing or unloadable)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise OSError(f"libkvc.so not found at {p}: build it with `python -m sparse_decode_attention_window_b200.build`")
    lib = ctypes.CDLL(p)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    f32 = ctypes.c_float
    sh = ctypes.POINTER(KvcShape)
    sig = {
        "kvc_score": (i32, [sh, vp, vp, vp, i32, vp, vp, vp, sz, vp]),
        "kvc_select": (i32, [sh, vp, vp, vp, f32, vp, vp, i32, vp, i32, vp, vp, sz, vp]),
        "kvc_alloc_budgets": (i32, [vp, i32, i32, i32, i32, i32, vp, vp, vp]),
        "kvc_layout": (i32, [vp, i32, i32, vp, vp, vp]),
        "kvc_compact": (i32, [sh, vp, vp, vp, i32, vp, vp, vp, vp, i64, vp, vp]),
        "kvc_layout_compact": (i32, [sh, vp, vp, vp, i32, vp, i32, vp, vp, vp, vp, i64, vp, vp]),
        "kvc_append": (i32, [sh, vp, vp, vp, vp, vp, vp, vp, i64, vp]),
        "kvc_append_window": (i32, [sh, vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, vp]),
        "kvc_decode_attn": (i32, [sh, vp, vp, vp, vp, vp, i64, vp, vp, sz, vp]),
        "kvc_workspace_size": (sz, [ctypes.c_int, sh, i32]),
        "kvc_get_status": (i32, [vp]),
        "kvc_last_error": (ctypes.c_char_p, []),
        "kvc_version": (ctypes.c_char_p, []),
        "kvc_launch_count": (ctypes.c_ulonglong, []),
        "kvc_decode_attn_noalloc": (i32, [sh, vp, vp, vp, vp, vp, i64, vp, vp]),
        "kvc_append_decode": (i32, [sh, vp, vp, vp, vp, vp, vp, vp, vp, i64, vp, vp, sz, vp]),
        "kvc_append_decode_chain": (i32, [sh, vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, vp, vp, sz, vp]),
        "kvc_select_chunks": (i32, [sh, vp, vp, i32, vp, i32, vp, i32, vp, vp]),
        "kvc_retained_mass": (i32, [sh, vp, i32, vp, i32, vp, vp, vp]),
        "kvc_profile_heads": (i32, [sh, vp, vp, i32, f32, vp, vp, vp]),
        "kvc_check_wait_limit": (i32, [i32, vp]),
        "kvc_diag_set_path": (i32, [i32, i32]),
        "kvc_diag_get_path": (i32, [i32]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib
