"""ctypes binding of ``libnvfp4.so`` (the C ABI declared in include/nvfp4.h).

Argument marshalling only.  The library is loaded from this package directory;
if it is missing the import of any entry point raises -- there is no CPU or
PyTorch fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4.so")

NVFP4_OK = 0
NVFP4_ERR_INVALID_ARG = 1
NVFP4_ERR_ALIGNMENT = 2
NVFP4_ERR_UNSUPPORTED_SHAPE = 3
NVFP4_ERR_CUDA = 4
NVFP4_ERR_TIMEOUT = 5
NVFP4_ERR_DEVICE = 6

SF_LINEAR = 0
SF_TCGEN05 = 1

MAX_SEGMENTS = 16
GLOBAL_SCALE_WORKSPACE_BYTES = 256
NOALLOC_SCRATCH_BYTES = 256

# Every symbol include/nvfp4.h declares, with (restype, argtypes).
P = ctypes.c_void_p
I64 = ctypes.c_int64
I32 = ctypes.c_int
ST = ctypes.c_int


class Segment(ctypes.Structure):
    _fields_ = [("n_offset", ctypes.c_int64), ("n_size", ctypes.c_int64),
                ("w_gscale", ctypes.c_void_p)]


class SegmentAct(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("a_log", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p)]


ACT_NONE, ACT_DECAY_GATE, ACT_SIGMOID = 0, 1, 2

SIGNATURES = {
    "nvfp4_global_scale": (ST, [P, I64, I64, I64, P, P, P, P]),
    "nvfp4_global_scale_noalloc": (ST, [P, I64, I64, I64, P, P, P]),
    "nvfp4_sf_bytes": (ST, [I64, I64, I32, ctypes.POINTER(ctypes.c_size_t)]),
    "nvfp4_quantize": (ST, [P, I64, I64, I64, P, P, P, I32, P]),
    "nvfp4_quantize_slice": (ST, [P, I64, I64, I64, P, P, P, I32, I64, I64, P]),
    "nvfp4_gemm": (ST, [P, P, P, P, P, P, P, I64, I64, I64, I64, P]),
    "nvfp4_fused_gemm": (ST, [P, P, P, P, P, ctypes.POINTER(Segment), I32, P, I64, I64, I64, P]),
    "nvfp4_fused_gemm_act": (ST, [P, P, P, P, P, ctypes.POINTER(Segment), ctypes.POINTER(SegmentAct),
                                  I32, P, I64, I64, I64, P]),
    "nvfp4_silu_mul": (ST, [P, I64, I64, I64, P, I64, P]),
    "nvfp4_fused_linear_host": (ST, [P, I64, I64, P, P, ctypes.POINTER(Segment), I32, P, P, P, P, P,
                                     P, P, P, P]),
    "nvfp4_fused_linear_host_overlap": (ST, [P, I64, I64, P, P, ctypes.POINTER(Segment), I32, P, P, P,
                                             P, P, P, P, P, P, P]),
    "nvfp4_gemm_silu_mul": (ST, [P, P, P, P, P, P, P, I64, I64, I64, I64, P, P, P, P]),
    "nvfp4_harmonize_scales": (ST, [P, I64, ctypes.POINTER(Segment), I32, I32, P, P]),
    "nvfp4_kv_scale_from_amax": (ST, [P, P, P]),
    "nvfp4_kv_quantize_e4m3": (ST, [P, I64, I64, I64, P, P, I64, P]),
    "nvfp4_last_device_status": (ST, [P]),
    "nvfp4_debug_wait_timeout": (ST, [I64, P]),
    "nvfp4_status_string": (ctypes.c_char_p, [ST]),
    "nvfp4_version": (ctypes.c_int, []),
}

_lib = None


class Nvfp4Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = lib().nvfp4_status_string(status).decode() if _lib is not None else str(status)
        super().__init__(f"{fn} failed: {msg} (status {status})")


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m nvfp4_w4a4_quantized_09_b200.build` (there is no fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def check(fn: str, status: int) -> None:
    if status != NVFP4_OK:
        raise Nvfp4Error(fn, status)
