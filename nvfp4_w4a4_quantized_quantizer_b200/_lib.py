"""ctypes declarations of the C ABI in include/nvfp4.h (libnvfp4.so, in-tree).

Loading fails loudly when the library has not been built: there is no CPU
fallback for any entry point.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnvfp4.so")

OK = 0
STATUS_NAMES = {0: "NVFP4_OK", -1: "NVFP4_ERR_INVALID_ARG", -2: "NVFP4_ERR_ALIGNMENT",
                -3: "NVFP4_ERR_UNSUPPORTED_SHAPE", -4: "NVFP4_ERR_CUDA", -5: "NVFP4_ERR_TIMEOUT",
                -6: "NVFP4_ERR_UNSUPPORTED_DEVICE"}
OP_NONE, OP_SIGMOID, OP_GDN_DECAY = 0, 1, 2
OUT_BF16, OUT_FP32 = 0, 1
MAX_SEGMENTS = 32

# Every symbol include/nvfp4.h declares, with (restype, argtypes).
_vp, _i64, _i32, _u64, _f32, _sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                    ctypes.c_uint64, ctypes.c_float, ctypes.c_size_t)
_st = ctypes.c_int


class Segment(ctypes.Structure):
    """nvfp4_segment."""
    _fields_ = [("n_offset", ctypes.c_int64), ("w_gs", ctypes.c_float), ("a_gs", ctypes.c_float),
                ("op", ctypes.c_int32), ("a_log", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p)]


SIGNATURES = {
    "nvfp4_codes_bytes": (_sz, [_i64, _i64]),
    "nvfp4_scale_bytes": (_sz, [_i64, _i64]),
    "nvfp4_global_scale": (_f32, [_f32]),
    "nvfp4_amax": (_st, [_vp, _i64, _i64, _i64, _vp, _vp]),
    "nvfp4_quantize_act": (_st, [_vp, _i64, _i64, _i64, _f32, _vp, _vp, _vp]),
    "nvfp4_quantize_weight_workspace_bytes": (_sz, [_i32]),
    "nvfp4_quantize_weight": (_st, [_vp, _i64, _i64, _i64, _vp, _i32, _vp, _vp, _vp, _vp, _vp]),
    "nvfp4_quantize_weight_noalloc": (_st, [_vp, _i64, _i64, _i64, _vp, _i32, _vp, _vp, _vp, _vp]),
    "nvfp4_noalloc_max_segments": (_i32, []),
    "nvfp4_linear": (_st, [_vp, _vp, _f32, _vp, _vp, _f32, _i64, _i64, _i64, _vp, _i64, _st, _vp]),
    "nvfp4_fused_linear": (_st, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, ctypes.POINTER(Segment), _i32,
                                 _vp, _i64, _st, _vp]),
    "nvfp4_gemm_workspace_bytes": (_sz, []),
    "nvfp4_fused_linear_ws": (_st, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, ctypes.POINTER(Segment),
                                    _i32, _vp, _i64, _st, _vp, _sz, _vp]),
    "nvfp4_gate_up_silu_quantize": (_st, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _f32, _f32, _f32,
                                          _f32, _vp, _vp, _vp]),
    "nvfp4_silu_mul": (_st, [_vp, _i64, _i64, _i64, _vp, _i64, _vp]),
    "nvfp4_kv_scale": (_f32, [_f32]),
    "nvfp4_kv_quantize_fp8": (_st, [_vp, _i64, _f32, _vp, _vp]),
    "nvfp4_gdn_recurrence": (_st, [_vp, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _vp, _vp, _vp]),
    "nvfp4_status_string": (ctypes.c_char_p, [_st]),
    "nvfp4_last_device_error": (_st, [_vp, ctypes.POINTER(ctypes.c_uint64)]),
    "nvfp4_set_gemm_path": (_st, [_i32]),
    "nvfp4_set_launch_overlap": (_st, [_i32]),
    "nvfp4_set_wait_limit_ns": (_st, [_u64]),
    "nvfp4_test_e2m1": (_st, [_vp, _vp, _i64, _vp]),
    "nvfp4_test_e4m3": (_st, [_vp, _vp, _i64, _vp]),
    "nvfp4_test_wait_timeout": (_st, [_u64, _vp]),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load libnvfp4.so (once).  Raises if it is missing or lacks a symbol."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m nvfp4_w4a4_quantized_quantizer_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)          # AttributeError if a declared symbol is not exported
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = load().nvfp4_status_string(status).decode()
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({msg})")


def check(status: int, where: str) -> None:
    if status != OK:
        raise NVFP4Error(status, where)
