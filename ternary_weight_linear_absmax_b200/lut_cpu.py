"""Host table-lookup BitLinear (ctypes binding of libbitlinear_lut_cpu.so,
include/bitlinear_lut_cpu.h).

The lookup-table contraction of "BitNet b1.58 — quantização ternária,
BitLinear, Zero-GEMM", section "Como o ecossistema bitnet.cpp acelera
inferência em CPUs e borda?": 81 pre-summed entries per block of 4 int8
activations, one table read per 4 ternary weights. Runs on the host CPU
(AVX-512, AVX2 or scalar, chosen at run time): the benchmark's second CPU
baseline. Arguments are numpy arrays; this module only marshals them.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbitlinear_lut_cpu.so")
ISA_AUTO, ISA_SCALAR, ISA_AVX2, ISA_AVX512 = 0, 1, 2, 3
ISA_NAMES = {ISA_SCALAR: "scalar", ISA_AVX2: "avx2", ISA_AVX512: "avx512"}
_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} not built; run `python -m ternary_weight_linear_absmax_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, vp, i64, i32, f32 = ctypes.POINTER, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        L.blc_best_isa.restype = i32
        L.blc_best_isa.argtypes = []
        L.blc_lut_index_bytes.restype = ctypes.c_size_t
        L.blc_lut_index_bytes.argtypes = [i64, i64]
        L.blc_lut_index_from_packed.restype = i64
        L.blc_lut_index_from_packed.argtypes = [vp, i64, i64, vp]
        L.blc_lut_table.restype = None
        L.blc_lut_table.argtypes = [vp, vp]
        L.blc_lut_gemm.restype = i32
        L.blc_lut_gemm.argtypes = [vp, i64, i64, vp, i64, vp, i32, i32]
        L.blc_bitlinear_lut.restype = i32
        L.blc_bitlinear_lut.argtypes = [vp, i64, i64, vp, f32, i64, f32, vp, vp, vp, i32, i32]
        _lib = L
    return _lib


def best_isa() -> int:
    return int(load().blc_best_isa())


def index_from_packed(W_packed: np.ndarray, K: int) -> np.ndarray:
    """2-bit packed [N, K/4] → LUT-indexed weights (uint8, 16-row blocks)."""
    W_packed = np.ascontiguousarray(W_packed, dtype=np.uint8)
    N = W_packed.shape[0]
    out = np.empty(int(load().blc_lut_index_bytes(N, K)), np.uint8)
    bad = load().blc_lut_index_from_packed(W_packed.ctypes.data, N, K, out.ctypes.data)
    if bad:
        raise ValueError(f"{bad} invalid 2-bit codes (3) in the packed weights")
    return out


def table(a4) -> np.ndarray:
    """The 81-entry table of one block of 4 int8 activations."""
    a = np.ascontiguousarray(a4, dtype=np.int8)
    assert a.shape == (4,)
    t = np.empty(81, np.int16)
    load().blc_lut_table(a.ctypes.data, t.ctypes.data)
    return t


def lut_gemm(A_q: np.ndarray, idx: np.ndarray, N: int, threads: int = 0,
             isa: int = ISA_AUTO) -> np.ndarray:
    """acc [M, N] int32 = A_q · W_qᵀ by table lookup."""
    A_q = np.ascontiguousarray(A_q, dtype=np.int8)
    M, K = A_q.shape
    acc = np.empty((M, N), np.int32)
    rc = load().blc_lut_gemm(A_q.ctypes.data, M, K, idx.ctypes.data, N, acc.ctypes.data,
                             int(threads), int(isa))
    if rc != 0:
        raise RuntimeError(f"instruction set {isa} not supported by this CPU")
    return acc


def bitlinear_lut(A: np.ndarray, idx: np.ndarray, gamma: float, N: int, eps: float = 1e-5,
                  threads: int = 0, isa: int = ISA_AUTO):
    """Host BitLinear forward: returns (Y fp32 [M, N], A_q, γ_A)."""
    A = np.ascontiguousarray(A, dtype=np.float32)
    M, K = A.shape
    Y = np.empty((M, N), np.float32)
    q = np.empty((M, K), np.int8)
    g = np.empty((M,), np.float32)
    rc = load().blc_bitlinear_lut(A.ctypes.data, M, K, idx.ctypes.data, float(np.float32(gamma)), N,
                                  float(np.float32(eps)), Y.ctypes.data, q.ctypes.data,
                                  g.ctypes.data, int(threads), int(isa))
    if rc != 0:
        raise RuntimeError(f"instruction set {isa} not supported by this CPU")
    return Y, q, g
