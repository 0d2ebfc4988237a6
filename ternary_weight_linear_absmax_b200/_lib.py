"""ctypes loader for libbitlinear.so (the C ABI in include/bitlinear.h).

Loading fails loudly when the in-tree library is missing: there is no
fallback implementation of any operation.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbitlinear.so")

BL_OK = 0
STATUS_NAMES = {
    0: "BL_OK", 1: "BL_ERR_INVALID_ARG", 2: "BL_ERR_SHAPE", 3: "BL_ERR_ALIGN",
    4: "BL_ERR_DTYPE", 5: "BL_ERR_CUDA", 6: "BL_ERR_TIMEOUT", 7: "BL_ERR_UNSUPPORTED",
    8: "BL_ERR_WORKSPACE",
}
BL_F32, BL_BF16 = 0, 1
BL_FLAG_PDL = 1
BL_FLAG_RAW_I32 = 2

class BlTaps(ctypes.Structure):
    """bl_taps of include/bitlinear.h: device pointers (0 = tap off)."""
    _fields_ = [("act_q", ctypes.c_void_p), ("act_gamma", ctypes.c_void_p),
                ("act_rowsum", ctypes.c_void_p), ("acc_up", ctypes.c_void_p),
                ("req_q", ctypes.c_void_p), ("req_gamma", ctypes.c_void_p),
                ("req_rowsum", ctypes.c_void_p), ("cta", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


# Every symbol declared in include/bitlinear.h: name -> (restype, argtypes).
_vp, _i64, _f32, _int, _uint, _sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_float,
                                     ctypes.c_int, ctypes.c_uint, ctypes.c_size_t)
SIGNATURES = {
    "bl_status_string": (ctypes.c_char_p, [_int]),
    "bl_version": (_int, []),
    "bl_gemv_max_tokens": (_int, []),
    "bl_contraction_path": (_int, [_i64, _i64, _i64, _int, _sz]),
    "bl_quant_weights_workspace_bytes": (_sz, [_i64, _i64]),
    "bl_quant_weights": (_int, [_vp, _int, _i64, _i64, _f32, _vp, _vp, _vp, _sz, _vp]),
    "bl_quant_acts": (_int, [_vp, _int, _i64, _i64, _f32, _vp, _vp, _vp, _vp]),
    "bl_zero_gemm_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "bl_zero_gemm": (_int, [_vp, _i64, _i64, _vp, _i64, _vp, _vp, _sz, _vp]),
    "bl_linear_q_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "bl_linear_q": (_int, [_vp, _vp, _vp, _i64, _i64, _vp, _vp, _i64, _int, _vp, _int, _vp,
                           _sz, _vp]),
    "bl_linear_q_ex": (_int, [_vp, _vp, _vp, _i64, _i64, _vp, _vp, _i64, _int, _vp, _int, _vp,
                              _sz, _uint, _vp]),
    "bl_linear_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "bl_linear": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _i64, _f32, _int, _vp, _int, _vp,
                         _sz, _vp]),
    "bl_linear_ex": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _i64, _f32, _int, _vp, _int, _vp,
                            _sz, _uint, _vp]),
    "bl_linear_taps": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _i64, _f32, _int, _vp, _int,
                              _vp, _sz, _uint, ctypes.POINTER(BlTaps), _vp]),
    "bl_linear_noalloc": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _i64, _f32, _int, _vp, _int,
                                 _vp]),
    "bl_ffn_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "bl_ffn_relu2": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _f32, _vp, _int,
                            _vp, _sz, _vp]),
    "bl_ffn_relu2_ex": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _f32, _vp, _int,
                               _vp, _sz, _uint, _vp]),
    "bl_ffn_relu2_taps": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _f32, _vp,
                                 _int, _vp, _sz, ctypes.POINTER(BlTaps), _vp]),
    "bl_radix3_row_bytes": (_i64, [_i64]),
    "bl_pack_radix3": (_int, [_vp, _i64, _i64, _vp, _vp]),
    "bl_linear_radix3": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _i64, _f32, _int, _vp, _int, _uint,
                                _vp]),
    "bl_pack_lut_index": (_int, [_vp, _i64, _i64, _vp, _vp]),
    "bl_linear_lut": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _i64, _f32, _vp, _int, _uint, _vp]),
    "bl_ffn_tp_up_workspace_bytes": (_sz, [_i64, _i64]),
    "bl_ffn_tp_up": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _vp, _f32, _vp, _vp, _vp, _vp, _sz,
                            _vp]),
    "bl_ffn_tp_down_workspace_bytes": (_sz, [_i64, _i64]),
    "bl_ffn_tp_down": (_int, [_vp, _vp, _vp, _vp, _i64, _i64, _vp, _i64, _f32, _vp, _vp, _sz,
                              _vp]),
    "bl_dequant_i32": (_int, [_vp, _vp, _vp, _i64, _i64, _int, _vp, _int, _vp]),
    "bl_ste_grad_input_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "bl_ste_grad_input": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _sz, _vp]),
    "bl_ste_grad_weight_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "bl_ste_grad_weight": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _i64, _vp, _int, _vp, _f32,
                                  _vp, _vp, _sz, _vp]),
    "bl_probe_pdl_floor": (_int, [_i64, _i64, _i64, _vp]),
    "bl_check_device_error": (_int, [_vp]),
    "bl_selftest_wait_timeout": (_int, [_i64, _vp]),
}

_lib = None


class BitLinearError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({status_string(status)})")


def load(path: str | None = None) -> ctypes.CDLL:
    """Load the library (once). Raises if it has not been built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(
            f"libbitlinear.so not found at {p}; build it with "
            "`python -m ternary_weight_linear_absmax_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    if path is None:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().bl_status_string(int(status)).decode()


def check(status: int, where: str) -> None:
    if status != BL_OK:
        raise BitLinearError(status, where)
