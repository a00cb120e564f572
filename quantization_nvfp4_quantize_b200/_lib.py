"""ctypes loader for ``libnvfp4_quads.so`` (the C ABI in include/nvfp4_quads.h).

No fallback: if the library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libnvfp4_quads.so")

c_void_p = ctypes.c_void_p
c_int32 = ctypes.c_int32
c_int64 = ctypes.c_int64
c_size_t = ctypes.c_size_t

# name -> (restype, argtypes), mirroring include/nvfp4_quads.h
SIGNATURES = {
    "nvfp4_version": (ctypes.c_int, []),
    "nvfp4_last_error_string": (ctypes.c_char_p, []),
    "nvfp4_read_status": (c_int32, [c_void_p, c_void_p, c_void_p]),
    "nvfp4_num_sms": (ctypes.c_int, []),
    "nvfp4_quantize_workspace_size": (c_size_t, [c_int64, c_int64]),
    "nvfp4_quantize": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p, c_void_p, c_void_p,
                                 c_void_p, c_int32, c_int64, c_void_p, c_void_p, c_void_p, c_int32, c_int32,
                                 c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "nvfp4_quantize_noalloc_max_scratch": (c_size_t, []),
    "nvfp4_quantize_noalloc": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p, c_void_p,
                                         c_void_p, c_void_p, c_int32, c_int64, c_void_p, c_void_p, c_void_p, c_int32,
                                         c_int32, c_void_p, c_void_p, c_void_p, c_void_p]),
    "nvfp4_qdq_workspace_size": (c_size_t, [c_int64, c_int64, c_int64]),
    "nvfp4_qdq_weights": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p, c_void_p,
                                    c_void_p, c_void_p, c_size_t, c_void_p]),
    "moe_route_workspace_size": (c_size_t, [c_int64, c_int32]),
    "moe_route": (c_int32, [c_void_p, c_int64, c_int32, c_int32, c_void_p, c_void_p, c_int32, c_void_p, c_void_p,
                            c_void_p, c_void_p, c_int64, c_void_p, c_size_t, c_void_p]),
    "nvfp4_gather_weight_channels": (c_int32, [c_void_p, c_void_p, c_int32, c_int64, c_int64, c_void_p,
                                               c_int32, c_int32, c_void_p, c_void_p]),
    "nvfp4_weights_channel_major": (c_int32, [c_void_p, c_void_p, c_int32, c_int64, c_int64, c_void_p, c_void_p,
                                              c_void_p]),
    "nvfp4_gather_weight_channels_cm": (c_int32, [c_void_p, c_void_p, c_int32, c_int64, c_int64, c_void_p,
                                                  c_int32, c_int32, c_void_p, c_void_p]),
    "moe_w4a4_grouped_gemm_rac": (c_int32, [c_void_p, c_void_p, c_void_p, c_int64, c_void_p, c_void_p,
                                            c_void_p, c_int64, c_int64, c_int32, c_void_p, c_int32, c_int32, c_void_p,
                                            c_void_p, c_int32, c_void_p, c_void_p, c_void_p, c_int64, c_void_p,
                                            c_void_p, c_void_p]),
    "moe_bf16_grouped_gemm": (c_int32, [c_void_p, c_int64, c_int64, c_void_p, c_int64, c_int64, c_int32, c_void_p,
                                        c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_int64, c_void_p, c_void_p,
                                        c_void_p]),
    "moe_gather_rows_bf16": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_int32, c_void_p, c_int64,
                                       c_int64, c_void_p]),
    "nvfp4_debug_encode": (c_int32, [c_void_p, c_int64, c_void_p, c_void_p, c_void_p]),
    "nvfp4_rac_residual_nvfp4_workspace_size": (c_size_t, []),
    "nvfp4_rac_residual_nvfp4": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p, c_void_p, c_int32,
                                           c_int32, c_void_p, c_int32, c_int64, c_void_p, c_void_p, c_void_p,
                                           c_size_t, c_void_p]),
    "fp8_quantize_workspace_size": (c_size_t, [c_int64]),
    "fp8_quantize": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_int64, c_void_p, c_void_p, c_void_p, c_void_p,
                               c_int32, c_int64, c_void_p, c_void_p, c_size_t, c_void_p]),
    "moe_w8a8_grouped_gemm": (c_int32, [c_void_p, c_void_p, c_int64, c_void_p, c_void_p, c_int64, c_int64, c_int32,
                                        c_void_p, c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_int64, c_void_p,
                                        c_void_p, c_void_p]),
    "nvfp4_quantize_experts_workspace_size": (c_size_t, [c_int64, c_int64, c_int32, c_int32]),
    "nvfp4_quantize_experts": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_int32, c_int32, c_void_p,
                                         c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int32, c_int32, c_void_p,
                                         c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "nvfp4_gather_weight_channels_cm_experts": (c_int32, [c_void_p, c_void_p, c_int32, c_int64, c_int64, c_void_p,
                                                          c_int32, c_int32, c_void_p, c_void_p]),
    "moe_routed_rows_bf16": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p, c_int64, c_int64,
                                       c_void_p]),
    "nvfp4_debug_gemm_wait_expiry": (c_int32, [c_void_p, c_void_p, c_void_p, c_int64, c_void_p, c_void_p, c_void_p,
                                               c_int64, c_int64, c_int32, c_void_p, c_int32, c_void_p, c_void_p,
                                               c_void_p, c_int64, c_void_p, c_int64, c_void_p]),
}

STATUS_NAMES = {0: "NVFP4_OK", 1: "NVFP4_ERR_INVALID_ARG", 2: "NVFP4_ERR_ALIGNMENT",
                3: "NVFP4_ERR_UNSUPPORTED_SHAPE", 4: "NVFP4_ERR_CUDA", 5: "NVFP4_ERR_TIMEOUT",
                6: "NVFP4_ERR_WORKSPACE"}

_lib = None


class Nvfp4Error(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def load() -> ctypes.CDLL:
    """Load the in-tree CUDA library (raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run __graft_entry__.build() or "
                               "python quantization_nvfp4_quantize_b200/build.py")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def check(status: int) -> None:
    if status != 0:
        msg = load().nvfp4_last_error_string()
        raise Nvfp4Error(status, msg.decode() if msg else "")
