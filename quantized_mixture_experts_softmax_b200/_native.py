"""ctypes loader for libmoe.so (the C ABI in include/moe.h).

There is no fallback: if the library is missing or cannot be loaded, importing this module
raises, and every call that the library rejects raises MoeError.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT", 6: "MOE_ERR_DEVICE_CHECK"}
MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE = 0, 1, 2, 3
MOE_ERR_CUDA, MOE_ERR_TIMEOUT, MOE_ERR_DEVICE_CHECK = 4, 5, 6

# Every symbol include/moe.h declares.
EXPORTS = [
    "moe_status_string", "moe_route", "moe_align_capacity", "moe_align_workspace_size", "moe_align",
    "moe_w4a16_workspace_size", "moe_w4a16_forward", "moe_blockfp8_workspace_size", "moe_blockfp8_forward",
    "moe_w4a16_gemm_workspace_size", "moe_w4a16_gemm", "moe_get_device_status", "moe_debug_wait_timeout",
    "moe_timing_enable", "moe_timing_read", "moe_align_noalloc", "moe_blockfp8_intermediate",
    "moe_w4a8_workspace_size", "moe_w4a8_forward", "moe_w4a8_intermediate",
]


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


class W4A16Args(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("topk_ids", ctypes.c_void_p), ("topk_w", ctypes.c_void_p),
                ("w13_q", ctypes.c_void_p), ("w13_s", ctypes.c_void_p), ("w2_q", ctypes.c_void_p),
                ("w2_s", ctypes.c_void_p), ("T", ctypes.c_int), ("H", ctypes.c_int), ("I", ctypes.c_int),
                ("E", ctypes.c_int), ("k", ctypes.c_int), ("out", ctypes.c_void_p), ("out_fp32", ctypes.c_int)]


class BlockFP8Args(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("xs", ctypes.c_void_p), ("topk_ids", ctypes.c_void_p),
                ("topk_w", ctypes.c_void_p), ("w13", ctypes.c_void_p), ("w13_s", ctypes.c_void_p),
                ("w2", ctypes.c_void_p), ("w2_s", ctypes.c_void_p), ("T", ctypes.c_int), ("H", ctypes.c_int),
                ("I", ctypes.c_int), ("E", ctypes.c_int), ("k", ctypes.c_int), ("out", ctypes.c_void_p),
                ("out_fp32", ctypes.c_int)]


class W4A8Args(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("topk_ids", ctypes.c_void_p), ("topk_w", ctypes.c_void_p),
                ("w13", ctypes.c_void_p), ("w13_sf", ctypes.c_void_p), ("w2", ctypes.c_void_p),
                ("w2_sf", ctypes.c_void_p), ("T", ctypes.c_int), ("H", ctypes.c_int), ("I", ctypes.c_int),
                ("E", ctypes.c_int), ("k", ctypes.c_int), ("out", ctypes.c_void_p), ("out_fp32", ctypes.c_int)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -c 'import __graft_entry__ as g; g.build()'` "
                          "(there is no fallback implementation)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_status_string.argtypes = [i32]
    L.moe_route.restype = i32
    L.moe_route.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp]
    L.moe_align_capacity.restype = sz
    L.moe_align_capacity.argtypes = [i32, i32, i32, i32]
    L.moe_align_workspace_size.restype = sz
    L.moe_align_workspace_size.argtypes = [i32, i32, i32]
    L.moe_align.restype = i32
    L.moe_align.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, sz, vp]
    L.moe_align_noalloc.restype = i32
    L.moe_align_noalloc.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp]
    L.moe_w4a16_workspace_size.restype = sz
    L.moe_w4a16_workspace_size.argtypes = [i32, i32, i32, i32, i32]
    L.moe_w4a16_forward.restype = i32
    L.moe_w4a16_forward.argtypes = [ctypes.POINTER(W4A16Args), vp, sz, vp]
    L.moe_blockfp8_workspace_size.restype = sz
    L.moe_blockfp8_workspace_size.argtypes = [i32, i32, i32, i32, i32]
    L.moe_blockfp8_forward.restype = i32
    L.moe_blockfp8_forward.argtypes = [ctypes.POINTER(BlockFP8Args), vp, sz, vp]
    L.moe_w4a8_workspace_size.restype = sz
    L.moe_w4a8_workspace_size.argtypes = [i32, i32, i32, i32, i32]
    L.moe_w4a8_forward.restype = i32
    L.moe_w4a8_forward.argtypes = [ctypes.POINTER(W4A8Args), vp, sz, vp]
    L.moe_w4a8_intermediate.restype = i32
    L.moe_w4a8_intermediate.argtypes = [vp, i32, i32, i32, i32, i32, ctypes.POINTER(vp), ctypes.POINTER(vp),
                                        ctypes.POINTER(vp)]
    L.moe_blockfp8_intermediate.restype = i32
    L.moe_blockfp8_intermediate.argtypes = [vp, i32, i32, i32, i32, i32, ctypes.POINTER(vp), ctypes.POINTER(vp),
                                            ctypes.POINTER(vp)]
    L.moe_w4a16_gemm_workspace_size.restype = sz
    L.moe_w4a16_gemm_workspace_size.argtypes = [i32, i32, i32, i32]
    L.moe_w4a16_gemm.restype = i32
    L.moe_w4a16_gemm.argtypes = [vp, i32, vp, vp, vp, i32, i32, i32, i32, vp, i32, vp, sz, vp]
    L.moe_get_device_status.restype = i32
    L.moe_get_device_status.argtypes = [vp]
    L.moe_debug_wait_timeout.restype = i32
    L.moe_debug_wait_timeout.argtypes = [i64, vp]
    L.moe_timing_enable.restype = i32
    L.moe_timing_enable.argtypes = [i32]
    L.moe_timing_read.restype = i32
    L.moe_timing_read.argtypes = [ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_double),
                                  ctypes.POINTER(ctypes.c_int), i32]
    return L


lib = _load()


def check(code: int, where: str) -> None:
    if code != MOE_OK:
        raise MoeError(code, where)
