"""ctypes loader for libqlora_b200.so (argument marshalling only).

Every compute step runs in the library's CUDA kernels; if the shared library
is missing this module raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_double, c_float, c_int, c_int32, c_int64, c_size_t, c_uint8, c_uint16, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqlora_b200.so")

STATUS = {
    0: "QLORA_OK", 1: "QLORA_ERR_NULL", 2: "QLORA_ERR_SHAPE", 3: "QLORA_ERR_ALIGN", 4: "QLORA_ERR_DTYPE",
    5: "QLORA_ERR_UNSUPPORTED", 6: "QLORA_ERR_CUDA", 7: "QLORA_ERR_WORKSPACE", 8: "QLORA_ERR_NONFINITE",
    9: "QLORA_ERR_TIMEOUT",
}
DTYPE_BF16, DTYPE_F32 = 0, 1


class NF4QConfig(ctypes.Structure):
    _fields_ = [("blocksize", c_int32), ("double_quant", c_int32), ("dq_blocksize", c_int32)]


class QLoraWeight(ctypes.Structure):
    _fields_ = [("out", c_int64), ("in_", c_int64), ("q", NF4QConfig), ("is_bf16", c_int32),
                ("codes", c_void_p), ("absmax", c_void_p), ("absmax_q", c_void_p), ("absmax2", c_void_p),
                ("w_bf16", c_void_p)]


# name -> (restype, argtypes); every symbol declared in include/qlora_b200.h
SIGNATURES = {
    "qlora_status_str": (c_char_p, [c_int]),
    "qlora_read_status": (c_int, [c_void_p, c_void_p]),
    "qlora_reset_status": (c_int, [c_void_p, c_void_p]),
    "qlora_reset_workspace": (c_int, [c_void_p, c_size_t, c_void_p]),
    "qlora_device_check": (c_int, [c_int]),
    "qlora_profile_events": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p]),
    "qlora_pair_clusters": (c_int32, []),
    "qlora_pair_schedule": (c_int, [c_int32, c_int32, c_int32, c_int32, c_void_p]),
    "nf4_rank_errors": (c_int, [c_int32, c_void_p, c_int32, c_void_p, c_void_p, c_void_p]),
    "nf4_quantize_workspace_size": (c_size_t, [c_int64]),
    "nf4_quantize": (c_int, [c_void_p, c_int32, c_int64, c_int64, NF4QConfig, c_void_p, c_void_p, c_void_p,
                             c_void_p, c_void_p, c_size_t, c_void_p]),
    "nf4_quantize_batch": (c_int, [c_int32, POINTER(c_void_p), POINTER(c_int64), c_int32, NF4QConfig,
                                   POINTER(c_void_p), POINTER(c_void_p), POINTER(c_void_p), POINTER(c_void_p),
                                   c_void_p, c_size_t, c_void_p]),
    "nf4_dequantize": (c_int, [POINTER(QLoraWeight), c_void_p, c_void_p]),
    "qlora_lora_merge": (c_int, [POINTER(QLoraWeight), c_void_p, c_void_p, c_int32, c_float, c_void_p, c_void_p]),
    "qlora_lora_merge_requantize_workspace_size": (c_size_t, [c_int64, c_int64]),
    "qlora_lora_merge_requantize": (c_int, [POINTER(QLoraWeight), c_void_p, c_void_p, c_int32, c_float, NF4QConfig,
                                            c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "qlora_fwd_workspace_size": (c_size_t, [c_int64, c_int64, c_int64, c_int32]),
    "qlora_bwd_workspace_size": (c_size_t, [c_int64, c_int64, c_int64, c_int32]),
    "qlora_linear_fwd": (c_int, [POINTER(QLoraWeight), c_void_p, c_int64, c_void_p, c_void_p, c_int32, c_float,
                                 c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "qlora_lora_down_workspace_size": (c_size_t, [c_int64, c_int64, c_int32]),
    "qlora_lora_down": (c_int, [c_void_p, c_int64, c_int64, c_void_p, c_int32, c_void_p, c_void_p, c_size_t, c_void_p]),
    "qlora_linear_fwd_t": (c_int, [POINTER(QLoraWeight), c_void_p, c_int64, c_void_p, c_void_p, c_int32, c_float,
                                   c_void_p, c_void_p, c_size_t, c_void_p]),
    "qlora_linear_bwd": (c_int, [POINTER(QLoraWeight), c_void_p, c_void_p, c_int64, c_void_p, c_void_p, c_int32,
                                 c_float, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "nf4_layer_error_rank_workspace_size": (c_size_t, [c_int32, POINTER(c_int64)]),
    "nf4_layer_error_rank": (c_int, [c_int32, POINTER(c_void_p), POINTER(c_int64), c_int32, NF4QConfig, c_int32,
                                     c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "nf4_layer_error_rank_budget": (c_int, [c_int32, POINTER(c_void_p), POINTER(c_int64), c_int32, NF4QConfig,
                                            c_int64, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                            c_void_p]),
    "nf4_k_from_fraction": (c_int, [c_int64, c_int64, c_int32, POINTER(c_int32)]),
    "nf4_quantize_residual_workspace_size": (c_size_t, [c_int64]),
    "nf4_quantize_residual": (c_int, [c_void_p, POINTER(QLoraWeight), NF4QConfig, c_void_p, c_void_p, c_void_p,
                                      c_void_p, c_void_p, c_size_t, c_void_p]),
    "nf4_dequantize_two_stage": (c_int, [POINTER(QLoraWeight), POINTER(QLoraWeight), c_void_p, c_void_p]),
    "nf4_layer_error_rank_noalloc": (c_int, [c_int32, POINTER(c_void_p), POINTER(c_int64), c_int32, NF4QConfig,
                                             c_int32, c_void_p, c_void_p, c_void_p, c_void_p]),
    "nf4_quantize_error_rank": (c_int, [c_int32, POINTER(c_void_p), POINTER(c_int64), c_int32, NF4QConfig, c_int32,
                                        POINTER(c_void_p), POINTER(c_void_p), POINTER(c_void_p), POINTER(c_void_p),
                                        c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
}

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libqlora_b200.so not built ({path}); run `python -m quantized_lora_fine_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class QLoraError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


def check(code: int, where: str) -> None:
    if code != 0:
        raise QLoraError(code, where)
