"""ctypes loader and signatures for librb.so (the C ABI in include/rb_api.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of the shared library. Loading fails loudly when the library is
missing; there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librb.so")

RB_OK = 0
STATUS_NAMES = {0: "RB_OK", 1: "RB_ERR_INVALID_ARG", 2: "RB_ERR_UNSUPPORTED", 3: "RB_ERR_ALIGNMENT",
                4: "RB_ERR_WORKSPACE", 5: "RB_ERR_CUDA", 6: "RB_ERR_DEVICE"}
RB_F32, RB_F16 = 0, 1
RB_ROWS, RB_SLICED = 0, 1

# every symbol include/rb_api.h declares
EXPORTED = ("rb_planes_words", "rb_scales_count", "rb_status_string", "rb_last_error",
            "rb_pack", "rb_gemv", "rb_gemv_workspace_bytes", "rb_gemv_grouped",
            "rb_gemv_grouped_workspace_bytes", "rb_gemv_check", "rb_gemv_noalloc",
            "rb_gemm", "rb_gemm_workspace_bytes", "rb_gemm_check",
            "rb_pack_fixed", "rb_dual_gemv", "rb_dual_gemv_workspace_bytes", "rb_gemm_reconstruct",
            "rb_gemv_swiglu", "rb_gemv_swiglu_workspace_bytes", "rb_gemm_from_weight",
            "rb_gemm_from_weight_workspace_bytes")


class RbError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {detail}")


class Layout(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int64), ("K", ctypes.c_int64),
                ("n_paths", ctypes.c_int32), ("group", ctypes.c_int32),
                ("order", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class GemvDesc(ctypes.Structure):
    _fields_ = [("planes", ctypes.c_void_p), ("alpha", ctypes.c_void_p),
                ("x", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("M", ctypes.c_int64), ("K", ctypes.c_int64)]


_lock = threading.Lock()
_lib = None


def load() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m residual_binary_weight_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
        st = ctypes.c_int
        lib.rb_planes_words.argtypes = [Layout]
        lib.rb_planes_words.restype = sz
        lib.rb_scales_count.argtypes = [Layout]
        lib.rb_scales_count.restype = sz
        lib.rb_status_string.argtypes = [st]
        lib.rb_status_string.restype = ctypes.c_char_p
        lib.rb_last_error.argtypes = []
        lib.rb_last_error.restype = ctypes.c_char_p
        lib.rb_pack.argtypes = [vp, st, i64, Layout, vp, vp, vp, vp]
        lib.rb_pack.restype = st
        lib.rb_gemv.argtypes = [vp, vp, st, Layout, vp, i64, i32, vp, st, i64, vp, sz, vp]
        lib.rb_gemv.restype = st
        lib.rb_gemv_workspace_bytes.argtypes = [Layout, i32]
        lib.rb_gemv_workspace_bytes.restype = sz
        lib.rb_gemv_swiglu.argtypes = [vp, vp, st, Layout, vp, i64, i32, vp, st, i64, vp, sz, vp]
        lib.rb_gemv_swiglu.restype = st
        lib.rb_gemv_swiglu_workspace_bytes.argtypes = [Layout, i32]
        lib.rb_gemv_swiglu_workspace_bytes.restype = sz
        lib.rb_gemm_from_weight.argtypes = [vp, st, i64, Layout, vp, i64, i32, vp, st, i64, vp, sz, vp]
        lib.rb_gemm_from_weight.restype = st
        lib.rb_gemm_from_weight_workspace_bytes.argtypes = [Layout, i32]
        lib.rb_gemm_from_weight_workspace_bytes.restype = sz
        lib.rb_gemv_grouped.argtypes = [vp, vp, i32, i32, i32, i32, st, st, i32, vp, sz, vp]
        lib.rb_gemv_grouped.restype = st
        lib.rb_gemv_grouped_workspace_bytes.argtypes = [vp, i32, i32, i32]
        lib.rb_gemv_grouped_workspace_bytes.restype = sz
        lib.rb_gemv_check.argtypes = [vp, vp]
        lib.rb_gemv_check.restype = st
        lib.rb_gemv_noalloc.argtypes = [vp, vp, st, Layout, vp, i64, i32, vp, st, i64, vp]
        lib.rb_gemv_noalloc.restype = st
        lib.rb_gemm.argtypes = [vp, vp, st, Layout, vp, i64, i32, vp, st, i64, vp, sz, vp]
        lib.rb_gemm.restype = st
        lib.rb_gemm_reconstruct.argtypes = [vp, vp, st, Layout, vp, i64, i32, vp, st, i64, vp, sz, vp]
        lib.rb_gemm_reconstruct.restype = st
        lib.rb_gemm_workspace_bytes.argtypes = [Layout, i32]
        lib.rb_gemm_workspace_bytes.restype = sz
        lib.rb_gemm_check.argtypes = [vp, vp]
        lib.rb_gemm_check.restype = st
        lib.rb_pack_fixed.argtypes = [vp, st, i64, Layout, vp, vp, vp, vp]
        lib.rb_pack_fixed.restype = st
        lib.rb_dual_gemv.argtypes = [vp, Layout, vp, vp, vp, i64, i32, vp, st, i64, vp, sz, vp]
        lib.rb_dual_gemv.restype = st
        lib.rb_dual_gemv_workspace_bytes.argtypes = [Layout, i32]
        lib.rb_dual_gemv_workspace_bytes.restype = sz
        _lib = lib
        return lib


def check(status: int) -> None:
    if status != RB_OK:
        detail = load().rb_last_error().decode(errors="replace")
        raise RbError(status, detail)
