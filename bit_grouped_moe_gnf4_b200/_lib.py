"""ctypes loader for libgnf4.so (the C ABI of include/gnf4.h).

Argument marshalling only. The library must have been built in-tree
(``python -m bit_grouped_moe_gnf4_b200.build``); if it is missing, importing
this module fails loudly -- there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgnf4.so")

GNF4_OK = 0
GNF4_ERR_INVALID_ARG = 1
GNF4_ERR_UNSUPPORTED_SHAPE = 2
GNF4_ERR_MISALIGNED = 3
GNF4_ERR_CUDA = 4
GNF4_ERR_DEVICE_STATUS = 5

GNF4_CHECK = 0x1
GNF4_FORCE_DECODE = 0x2
GNF4_FORCE_PREFILL = 0x4
GNF4_TEST_STALL = 0x100

GNF4_DTYPE_BF16 = 0
GNF4_DTYPE_F16 = 1
GNF4_DTYPE_F32 = 2

STATUS_NAMES = {0: "GNF4_OK", 1: "GNF4_ERR_INVALID_ARG", 2: "GNF4_ERR_UNSUPPORTED_SHAPE",
                3: "GNF4_ERR_MISALIGNED", 4: "GNF4_ERR_CUDA", 5: "GNF4_ERR_DEVICE_STATUS"}

# every symbol include/gnf4.h declares
EXPORTED = ("gnf4_last_error", "gnf4_version", "gnf4_quantize_nf4", "gnf4_quantize_mxfp4",
            "gnf4_grouped_gemm_nf4", "gnf4_grouped_gemm_mxfp4", "gnf4_grouped_gemm_launches",
            "gnf4_device_status", "gnf4_swiglu", "gnf4_combine_topk", "gnf4_dgrad_nf4",
            "gnf4_dgrad_mxfp4", "gnf4_routing_metadata", "gnf4_grouped_gemm_nf4_ex",
            "gnf4_grouped_gemm_mxfp4_ex", "gnf4_absmax_to_bf16", "gnf4_grouped_gemm_swiglu_nf4",
            "gnf4_grouped_gemm_swiglu_mxfp4")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python -m bit_grouped_moe_gnf4_b200.build` (nvcc, sm_100a)")

lib = ctypes.CDLL(LIB_PATH)

_p, _i64, _i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int

lib.gnf4_last_error.restype = ctypes.c_char_p
lib.gnf4_last_error.argtypes = []
lib.gnf4_version.restype = _i32
lib.gnf4_version.argtypes = []
for _name in ("gnf4_quantize_nf4", "gnf4_quantize_mxfp4"):
    getattr(lib, _name).restype = _i32
    getattr(lib, _name).argtypes = [_p, _i64, _i64, _p, _p, _p]
for _name in ("gnf4_grouped_gemm_nf4", "gnf4_grouped_gemm_mxfp4"):
    getattr(lib, _name).restype = _i32
    getattr(lib, _name).argtypes = [_p, _p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _i64, _i64,
                                    _p, _i32, _p]
lib.gnf4_grouped_gemm_nf4_ex.restype = _i32
lib.gnf4_grouped_gemm_nf4_ex.argtypes = [_p, _i32, _p, _p, _i32, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _i64,
                                         _i64, _p, _i32, _p]
lib.gnf4_grouped_gemm_mxfp4_ex.restype = _i32
lib.gnf4_grouped_gemm_mxfp4_ex.argtypes = [_p, _i32, _p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _i64,
                                           _i64, _p, _i32, _p]
lib.gnf4_grouped_gemm_swiglu_nf4.restype = _i32
lib.gnf4_grouped_gemm_swiglu_nf4.argtypes = lib.gnf4_grouped_gemm_nf4_ex.argtypes
lib.gnf4_grouped_gemm_swiglu_mxfp4.restype = _i32
lib.gnf4_grouped_gemm_swiglu_mxfp4.argtypes = lib.gnf4_grouped_gemm_mxfp4_ex.argtypes
lib.gnf4_absmax_to_bf16.restype = _i32
lib.gnf4_absmax_to_bf16.argtypes = [_p, _i64, _p, _p]
for _name in ("gnf4_dgrad_nf4", "gnf4_dgrad_mxfp4"):
    getattr(lib, _name).restype = _i32
    getattr(lib, _name).argtypes = [_p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _i64, _p, _i32, _p]
lib.gnf4_routing_metadata.restype = _i32
lib.gnf4_routing_metadata.argtypes = [_p, _p, _i64, _i64, _i64, _p, _p, _p, _p, _p]
lib.gnf4_swiglu.restype = _i32
lib.gnf4_swiglu.argtypes = [_p, _i64, _i64, _p, _p]
lib.gnf4_combine_topk.restype = _i32
lib.gnf4_combine_topk.argtypes = [_p, _i64, _i64, _p, _p, _i64, _i64, _p, _p]
lib.gnf4_device_status.restype = _i32
lib.gnf4_device_status.argtypes = [_p]
lib.gnf4_grouped_gemm_launches.restype = _i32
lib.gnf4_grouped_gemm_launches.argtypes = [_i64, _i32]


class Gnf4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lib.gnf4_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def check(status: int, where: str) -> None:
    if status != GNF4_OK:
        raise Gnf4Error(status, where)
