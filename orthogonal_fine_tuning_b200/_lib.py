"""ctypes declarations for liboft.so (the C ABI in include/oft.h)."""

from __future__ import annotations

import ctypes
import os

from .build import LIB_PATH

OFT_OK = 0
OFT_ERR_INVALID_ARG = 1
OFT_ERR_UNSUPPORTED = 2
OFT_ERR_CUDA = 3
OFT_ERR_TIMEOUT = 4
OFT_ERR_WORKSPACE = 5

OFT_W_INT4 = 1
OFT_W_FP8 = 2
OFT_W_MXFP4 = 3

OFT_NOALLOC_SCRATCH_BYTES = 32 << 20

EXPORTS = (
    "oft_version", "oft_last_error", "oft_check_device", "oft_build_rotation",
    "oft_linear_fwd_workspace", "oft_linear_fwd", "oft_linear_bwd_workspace", "oft_linear_bwd",
    "moe_chunked_oft_workspace", "moe_chunked_oft_fwd", "oft_dequant_weight", "oft_rotate",
    "oft_cayley_backward", "oft_debug_bounded_wait", "oft_profile_begin", "oft_profile_end",
    "oft_linear_fwd_noalloc", "oft_set_gemm_mode", "moe_fused_oft_workspace", "moe_fused_oft_fwd",
    "moe_chunked_oft_bwd_workspace", "moe_chunked_oft_bwd", "moe_chunked_oft_layer_workspace",
    "moe_chunked_oft_layer_fwd", "oft_linear_fwd_weight_side_workspace", "oft_linear_fwd_weight_side",
    "oft_gemm_schedule", "oft_moe_chunk_dequant",
)


class CWeight(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("d_in", ctypes.c_int), ("d_out", ctypes.c_int), ("group", ctypes.c_int),
                ("n_experts", ctypes.c_int)]


class CSplit(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int), ("sizes", ctypes.c_int * 4)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_Z = ctypes.c_size_t
_WP = ctypes.POINTER(CWeight)
_SP = ctypes.POINTER(CSplit)

_SIGS = {
    "oft_version": (ctypes.c_char_p, []),
    "oft_last_error": (ctypes.c_char_p, []),
    "oft_check_device": (_I, [_P]),
    "oft_build_rotation": (_I, [_P, _I, _I, _P, _P]),
    "oft_linear_fwd_workspace": (_Z, [_I, _WP, _SP, _I]),
    "oft_linear_fwd": (_I, [_P, _I, _WP, _SP, _I, _P, _P, _P, _Z, _P]),
    "oft_linear_fwd_weight_side_workspace": (_Z, [_WP]),
    "oft_linear_fwd_weight_side": (_I, [_P, _I, _WP, _SP, _I, _P, _P, _P, _Z, _P]),
    "oft_linear_bwd_workspace": (_Z, [_I, _WP, _SP, _I]),
    "oft_linear_bwd": (_I, [_P, _P, _I, _WP, _SP, _I, _P, _P, _P, _P, _Z, _P]),
    "moe_chunked_oft_workspace": (_Z, [_I, _I, _I, _I, _WP, _I]),
    "moe_chunked_oft_fwd": (_I, [_P, _I, _P, _I, _I, _I, _WP, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _P]),
    "moe_fused_oft_workspace": (_Z, [_I, _I, _I, _I, _WP, _I]),
    "moe_fused_oft_fwd": (_I, [_P, _I, _P, _I, _I, _I, _WP, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _P]),
    "moe_chunked_oft_bwd_workspace": (_Z, [_I, _I, _I, _I, _WP, _I]),
    "moe_chunked_oft_bwd": (_I, [_P, _P, _I, _P, _I, _I, _I, _WP, _I, _P, _P, _P, _P, _P, _Z, _P]),
    "moe_chunked_oft_layer_workspace": (_Z, [_I, _I, _I, _I, _WP, _WP, _I]),
    "moe_chunked_oft_layer_fwd": (_I, [_P, _I, _P, _I, _I, _I, _WP, _WP, _I, _P, _P, _P, _P, _Z, _P]),
    "oft_dequant_weight": (_I, [_WP, _P, _I, _P]),
    "oft_moe_chunk_dequant": (_I, [_WP, _P, _I, _I, _I, _P, _P]),
    "oft_rotate": (_I, [_P, _I, _I, _I, _I, _P, _P, _P]),
    "oft_cayley_backward": (_I, [_P, _P, _I, _I, _P, _P]),
    "oft_debug_bounded_wait": (_I, [_I, _P]),
    "oft_set_gemm_mode": (_I, [_I]),
    "oft_gemm_schedule": (_I, [_I, _P, _P, _P, _I, _I, _P, _P, _P]),
    "oft_linear_fwd_noalloc": (_I, [_P, _I, _WP, _SP, _I, _P, _P, _P]),
    "oft_profile_begin": (_I, [_I]),
    "oft_profile_end": (_I, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int), _I,
                            ctypes.POINTER(ctypes.c_int)]),
}

KERNEL_CLASSES = ("gemm", "rotate", "dequant", "cayley", "grad", "route")


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python orthogonal_fine_tuning_b200/build.py` "
            "(the OFT path has no CPU fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib
