"""ctypes declarations of libnvfp4moe.so (the C ABI in include/nvfp4moe.h).

There is no fallback: if the library is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnvfp4moe.so")

OK, INVALID_ARG, UNSUPPORTED_SHAPE, WORKSPACE_TOO_SMALL, CUDA_ERROR, DEVICE_FAULT = range(6)
SF_ROWMAJOR, SF_MMA = 0, 1
SCALE_GIVEN, SCALE_DYNAMIC = 0, 1
DTYPE_BF16, DTYPE_F32 = 0, 1
PATH_AUTO, PATH_GEMV, PATH_GEMM = 0, 1, 2
COMBINE_AUTO, COMBINE_ORDERED, COMBINE_ACCUMULATE = 0, 1, 2
ACT_NVFP4, ACT_BF16 = 0, 1
LAUNCH_AUTO, LAUNCH_SINGLE, LAUNCH_MULTI, LAUNCH_SINGLE_TILE, LAUNCH_SINGLE_LOCAL = 0, 1, 2, 3, 4
STAGES = 7
STAGE_NAMES = ("route", "permute", "quantize_x", "gate_up", "down", "combine")
DEV_BAD_EXPERT_ID, DEV_DUPLICATE_ID, DEV_ROW_OVERFLOW, DEV_TIMEOUT, DEV_BAD_GATHER = 1, 2, 4, 8, 16

STATUS_NAMES = {OK: "OK", INVALID_ARG: "INVALID_ARG", UNSUPPORTED_SHAPE: "UNSUPPORTED_SHAPE",
                WORKSPACE_TOO_SMALL: "WORKSPACE_TOO_SMALL", CUDA_ERROR: "CUDA_ERROR",
                DEVICE_FAULT: "DEVICE_FAULT"}


class Nvfp4MoeError(RuntimeError):
    def __init__(self, status: int, fn: str, msg: str):
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t


class MoeFfnDesc(ctypes.Structure):
    _fields_ = [
        ("T", _i32), ("H", _i32), ("I", _i32), ("E", _i32), ("top_k", _i32),
        ("path", _i32), ("x_scale_mode", _i32),
        ("x_scale", _vp),
        ("w13_codes", _vp), ("w13_sf", _vp), ("w13_scale", _vp),
        ("w2_codes", _vp), ("w2_sf", _vp), ("w2_scale", _vp),
        ("h_scale", _vp), ("h_amax", _vp), ("stage_events", _vp), ("combine", _i32), ("h_scale_mode", _i32),
        ("act_mode", _i32), ("shared_I", _i32), ("shared_w13", _vp), ("shared_w2", _vp), ("launch_mode", _i32),
    ]


class MoeFfnWsLayout(ctypes.Structure):
    _fields_ = [(n, _i64) for n in (
        "topk_ids", "topk_w", "counts", "offsets", "padded_offsets", "pair_to_row", "row_token",
        "row_pair", "tile_expert", "active", "x_scale", "x_codes", "x_sf", "h_codes", "h_sf",
        "slots", "amax_partials", "total", "x_rows", "h_rows", "items")] + [
        ("m_tile", _i32), ("path", _i32), ("combine", _i32), ("single_launch", _i32), ("h_f32", _i64), ("h_stats", _i64),
        ("h_bf16", _i64), ("shared_h", _i64), ("shared_y", _i64)]


# name -> (restype, argtypes)
SIGNATURES = {
    "nvfp4moe_last_error": (ctypes.c_char_p, []),
    "nvfp4moe_version": (_i32, []),
    "nvfp4moe_device_status": (_i32, [_vp, _i32, ctypes.POINTER(ctypes.c_uint32)]),
    "nvfp4_codec_convert": (_i32, [_vp, _i64, _vp, _vp, _vp]),
    "nvfp4_quantize_workspace_size": (_sz, [_i64, _i64, _i64]),
    "nvfp4_quantize": (_i32, [_vp, _i32, _i64, _i64, _i64, _i64, _i64, _vp, _i64, _i32, _vp, _vp,
                              _i64, _vp, _i64, _i32, _vp, _sz, _vp]),
    "nvfp4_quantize_dynamic_noalloc": (_i32, [_vp, _i32, _i64, _i64, _i64, _i64, _i64, _vp, _i64, _vp, _vp,
                                              _i64, _vp, _i64, _i32, _vp]),
    "nvfp4_from_mxfp4_workspace_size": (_sz, [_i64]),
    "nvfp4_from_mxfp4": (_i32, [_vp, _vp, _i64, _i64, _i64, _vp, _i64, _vp, _vp, _vp, _vp, _sz, _vp]),
    "nvfp4_prep_weights": (_i32, [_vp, _vp, _i32, _i64, _i64, _i64, _vp, _i64, _vp, _vp, _i32, _vp]),
    "moe_route": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moe_permute_rows_capacity": (_i64, [_i32, _i32, _i32, _i32]),
    "moe_permute": (_i32, [_vp, _i32, _i32, _i32, _i32, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                           _vp, _vp, _vp]),
    "nvfp4_gemm_workspace_size": (_sz, [_i64, _i64, _i64]),
    "nvfp4_gemm": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _i32, _vp, _sz, _vp]),
    "moe_ffn_workspace_layout": (_i32, [ctypes.POINTER(MoeFfnDesc), ctypes.POINTER(MoeFfnWsLayout)]),
    "moe_ffn_workspace_size": (_sz, [ctypes.POINTER(MoeFfnDesc)]),
    "moe_ffn_forward": (_i32, [ctypes.POINTER(MoeFfnDesc), _vp, _vp, _vp, _vp, _sz, _vp]),
    "nvfp4moe_mma_peak_probe": (_i32, [_i64, _vp]),
    "nvfp4moe_mma_peak_probe_flops": (_i64, [_i64]),
    "nvfp4moe_wait_selftest": (_i32, [ctypes.c_uint32, _vp, _vp]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Loads libnvfp4moe.so from the package directory (raises if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m nvfp4_mixture_experts_w4a4_b200.build`"
                " (there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def check(status: int, fn: str) -> None:
    if status != OK:
        msg = lib().nvfp4moe_last_error().decode(errors="replace")
        raise Nvfp4MoeError(status, fn, msg)
