"""ctypes binding of libkda.so (argument marshalling only; every step runs in the library)."""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
# KDA_LIB selects another build of the library (a variant from `build --define`); the default is
# the in-tree libkda.so.
LIB_PATH = os.environ.get("KDA_LIB") or os.path.join(PKG, "libkda.so")

# Every symbol include/kda.h declares.
EXPORTS = ("kda_status_string", "kda_plan_size", "kda_plan", "kda_workspace_size",
           "kda_forward", "kda_device_status", "kda_forward_noalloc", "kda_decode",
           "kda_plan_segmented", "kda_forward_summary", "kda_state_chain", "kda_noalloc_status")

STATUS = {0: "KDA_OK", 1: "KDA_ERR_NULL", 2: "KDA_ERR_LAYOUT", 3: "KDA_ERR_SHAPE",
          4: "KDA_ERR_HEADS", 5: "KDA_ERR_DIM", 6: "KDA_ERR_LOWER_BOUND", 7: "KDA_ERR_SEQLENS",
          8: "KDA_ERR_PLAN", 9: "KDA_ERR_ALIAS", 10: "KDA_ERR_WORKSPACE", 11: "KDA_ERR_CUDA",
          12: "KDA_ERR_TIMEOUT", 13: "KDA_ERR_DEVICE", 14: "KDA_ERR_ALIGN",
          15: "KDA_ERR_CAPACITY"}


class KdaShape(ctypes.Structure):
    _fields_ = [("layout", ctypes.c_int32), ("B", ctypes.c_int32), ("Nqk", ctypes.c_int32),
                ("Nv", ctypes.c_int32), ("S", ctypes.c_int32), ("D", ctypes.c_int32)]


class KdaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = int(code)
        self.name = STATUS.get(self.code, f"KDA_ERR_{code}")
        msg = load().kda_status_string(self.code).decode()
        super().__init__(f"{where}: {msg}")


_lib = None


def load():
    """Load libkda.so; raise loudly if it has not been built (there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m chunked_kda_prefill_b200.build` (needs nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    i32, sz, vp = ctypes.c_int32, ctypes.c_size_t, ctypes.c_void_p
    p_i32 = ctypes.POINTER(ctypes.c_int32)
    p_sz = ctypes.POINTER(ctypes.c_size_t)
    p_shape = ctypes.POINTER(KdaShape)
    L.kda_status_string.argtypes = [ctypes.c_int]
    L.kda_status_string.restype = ctypes.c_char_p
    L.kda_plan_size.argtypes = [p_shape, p_sz]
    L.kda_plan.argtypes = [p_shape, p_i32, i32, p_i32, sz]
    L.kda_workspace_size.argtypes = [p_i32, sz, p_sz]
    L.kda_forward.argtypes = [p_shape, p_i32, vp, sz, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp,
                              vp, ctypes.c_float, vp, sz, vp, vp, vp]
    L.kda_device_status.argtypes = [vp, vp]
    L.kda_forward_noalloc.argtypes = [p_shape, p_i32, vp, sz, vp, vp, vp, vp, vp, ctypes.c_float,
                                      vp, vp, vp, ctypes.c_float, vp, vp, vp]
    L.kda_noalloc_status.argtypes = [vp]
    L.kda_plan_segmented.argtypes = [p_shape, p_i32, i32, i32, p_i32, sz]
    L.kda_decode.argtypes = [i32, i32, i32, i32, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp,
                             ctypes.c_float, vp, vp, vp]
    L.kda_forward_summary.argtypes = [p_shape, p_i32, vp, sz, vp, vp, vp, vp, vp, vp, vp,
                                      ctypes.c_float, vp, sz, vp, vp, vp]
    L.kda_state_chain.argtypes = [i32, i32, i32, vp, vp, vp, ctypes.c_int64, vp, vp]
    for f in ("kda_plan_size", "kda_plan", "kda_workspace_size", "kda_forward",
              "kda_device_status", "kda_forward_noalloc", "kda_decode", "kda_plan_segmented",
              "kda_forward_summary", "kda_state_chain", "kda_noalloc_status"):
        getattr(L, f).restype = ctypes.c_int
    _lib = L
    return L


def check(code: int, where: str) -> None:
    if code != 0:
        raise KdaError(code, where)
