"""ctypes declarations of the libnvfp4 C ABI (include/nvfp4.h).

Loading is lazy: importing the package does not need the shared library, but
the first call of any operation does, and it raises if ``libnvfp4.so`` has not
been built (``python -m nvfp4_w4a4_quantized_08_b200.build``).  There is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libnvfp4.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED_SHAPE = 2
ERR_MISALIGNED = 3
ERR_WORKSPACE = 4
ERR_ARCH = 5
ERR_CUDA = 6
ERR_TIMEOUT = 7
ERR_DOMAIN = 8

BF16 = 0
FP32 = 1
SF_ROWMAJOR = 0
SF_MMA128x4 = 1
SCALE_ONTO_6 = 0
SCALE_FOUR_OVER_SIX = 1
ACT_NONE = 0
ACT_GELU_TANH = 1
KV_MAX_CHUNK_FRAMES = 8
KV_MAX_WINDOW_SLOTS = 256

EXPORTS = (
    "nvfp4_codes_bytes", "nvfp4_sf_bytes", "nvfp4_workspace_bytes", "nvfp4_quantize",
    "nvfp4_dequantize", "nvfp4_gemm", "nvfp4_kv_quant_chunk", "nvfp4_kv_dequant_window",
    "nvfp4_get_device_status", "nvfp4_set_wait_limit_ns", "nvfp4_status_string",
    "nvfp4_quantize_noalloc", "nvfp4_window_attention", "nvfp4_sink_plan_create",
    "nvfp4_sink_plan_destroy", "nvfp4_sink_plan_next", "nvfp4_sink_plan_frame_of_slot",
)


class Tensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("sf", ctypes.c_void_p), ("s_t", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("sf_layout", ctypes.c_int32)]


class KvCache(ctypes.Structure):
    _fields_ = [("k_codes", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
                ("k_sf", ctypes.c_void_p), ("v_sf", ctypes.c_void_p),
                ("k_st", ctypes.c_void_p), ("v_st", ctypes.c_void_p),
                ("n_slots", ctypes.c_int32), ("tokens_per_frame", ctypes.c_int32),
                ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("scale_rule", ctypes.c_int32)]


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"libnvfp4.so not found at {LIB_PATH}; build it with "
                "`python -m nvfp4_w4a4_quantized_08_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        i64, i32, vp, sz = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t
        TP = ctypes.POINTER(Tensor)
        KP = ctypes.POINTER(KvCache)
        L.nvfp4_codes_bytes.restype = sz
        L.nvfp4_codes_bytes.argtypes = [i64, i64]
        L.nvfp4_sf_bytes.restype = sz
        L.nvfp4_sf_bytes.argtypes = [i64, i64, i32]
        L.nvfp4_workspace_bytes.restype = sz
        L.nvfp4_workspace_bytes.argtypes = []
        L.nvfp4_quantize.restype = i32
        L.nvfp4_quantize.argtypes = [vp, i32, i64, i64, i64, TP, vp, vp, vp, sz, vp]
        L.nvfp4_quantize_noalloc.restype = i32
        L.nvfp4_quantize_noalloc.argtypes = [vp, i32, i64, i64, i64, TP, vp, vp]
        L.nvfp4_dequantize.restype = i32
        L.nvfp4_dequantize.argtypes = [TP, vp, i64, vp]
        L.nvfp4_gemm.restype = i32
        L.nvfp4_gemm.argtypes = [TP, TP, vp, i32, i64, i32, vp, i64, vp, sz, vp]
        L.nvfp4_kv_quant_chunk.restype = i32
        L.nvfp4_kv_quant_chunk.argtypes = [KP, vp, vp, i64, ctypes.POINTER(ctypes.c_int32), i32,
                                             vp, vp, vp, sz, vp]
        L.nvfp4_kv_dequant_window.restype = i32
        L.nvfp4_kv_dequant_window.argtypes = [KP, ctypes.POINTER(ctypes.c_int32), i32, vp, vp, vp]
        L.nvfp4_sink_plan_create.restype = vp
        L.nvfp4_sink_plan_create.argtypes = [i32, i32, i32, i32]
        L.nvfp4_sink_plan_destroy.restype = None
        L.nvfp4_sink_plan_destroy.argtypes = [vp]
        L.nvfp4_sink_plan_next.restype = i32
        L.nvfp4_sink_plan_next.argtypes = [vp, i32, i32, ctypes.POINTER(ctypes.c_int32),
                                           ctypes.POINTER(ctypes.c_int32),
                                           ctypes.POINTER(ctypes.c_int32)]
        L.nvfp4_sink_plan_frame_of_slot.restype = i64
        L.nvfp4_sink_plan_frame_of_slot.argtypes = [vp, i32]
        L.nvfp4_window_attention.restype = i32
        L.nvfp4_window_attention.argtypes = [KP, ctypes.POINTER(ctypes.c_int32), i32, vp, i64,
                                             i64, ctypes.c_float, vp, i64, vp, ctypes.c_size_t,
                                             vp]
        L.nvfp4_get_device_status.restype = i32
        L.nvfp4_get_device_status.argtypes = [vp, vp]
        L.nvfp4_set_wait_limit_ns.restype = None
        L.nvfp4_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        L.nvfp4_status_string.restype = ctypes.c_char_p
        L.nvfp4_status_string.argtypes = [i32]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().nvfp4_status_string(int(status)).decode()


def check(status: int, what: str) -> None:
    if status != OK:
        raise NVFP4Error(status, what)
