"""CPU oracle for the BitLinear forward pass (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: the independent reference the CUDA path is checked
against. Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg may import this package; the product path never does.

The arithmetic lives in ``bitlinear_oracle.cpp`` (plain C++, fp32 decisions,
double sums), each function citing the page section it follows:
"BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM" for the math and
"Arquitetura Hibrida Multimodal para bitnet.cpp" (utils/bit_layers.py) for
the API names. This wrapper only marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bitlinear_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "libbitlinear_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library with g++ (no fast-math, no FMA
    contraction) and return its path."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math",
           "-fopenmp", "-shared", "-fPIC", _SRC, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _p(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        i64, f32, i32 = ctypes.c_int64, ctypes.c_float, ctypes.c_int
        P = ctypes.POINTER
        L.orc_sum_abs.restype = ctypes.c_double
        L.orc_sum_abs.argtypes = [P(ctypes.c_float), i64]
        L.orc_absmean_gamma.restype = f32
        L.orc_absmean_gamma.argtypes = [P(ctypes.c_float), i64, i64]
        L.orc_ternary_codes.argtypes = [P(ctypes.c_float), i64, i64, f32, f32, P(ctypes.c_int8)]
        L.orc_quant_weights.restype = f32
        L.orc_quant_weights.argtypes = [P(ctypes.c_float), i64, i64, f32, P(ctypes.c_int8)]
        L.orc_pack_ternary.argtypes = [P(ctypes.c_int8), i64, i64, P(ctypes.c_uint8)]
        L.orc_unpack_ternary.restype = i64
        L.orc_unpack_ternary.argtypes = [P(ctypes.c_uint8), i64, i64, P(ctypes.c_int8)]
        L.orc_quant_acts.argtypes = [P(ctypes.c_float), i64, i64, f32, P(ctypes.c_int8), P(ctypes.c_float)]
        L.orc_zero_gemm.argtypes = [P(ctypes.c_int8), P(ctypes.c_int8), i64, i64, i64, P(ctypes.c_int32)]
        L.orc_lut_gemm.argtypes = [P(ctypes.c_int8), P(ctypes.c_int8), i64, i64, i64, P(ctypes.c_int32)]
        L.orc_dequant.argtypes = [P(ctypes.c_int32), P(ctypes.c_float), f32, i64, i64, i32, P(ctypes.c_double)]
        L.orc_dequant_f32.argtypes = [P(ctypes.c_int32), P(ctypes.c_float), f32, i64, i64, P(ctypes.c_float)]
        L.orc_relu2_requant.argtypes = [P(ctypes.c_int32), P(ctypes.c_float), f32, i64, i64, f32,
                                        P(ctypes.c_int8), P(ctypes.c_float)]
        L.orc_ste_grad_input.argtypes = [P(ctypes.c_float), i64, i64, P(ctypes.c_int8), i64, f32,
                                         P(ctypes.c_double)]
        L.orc_ste_weight_mask.argtypes = [P(ctypes.c_float), i64, i64, f32, f32, P(ctypes.c_uint8)]
        L.orc_ste_grad_weight.argtypes = [P(ctypes.c_float), i64, i64, P(ctypes.c_int8),
                                          P(ctypes.c_float), i64, P(ctypes.c_float), f32, f32,
                                          P(ctypes.c_double)]
        L.orc_radix3_row_bytes.restype = i64
        L.orc_radix3_row_bytes.argtypes = [i64]
        L.orc_pack_radix3.argtypes = [P(ctypes.c_int8), i64, i64, P(ctypes.c_uint8)]
        L.orc_unpack_radix3.restype = i64
        L.orc_unpack_radix3.argtypes = [P(ctypes.c_uint8), i64, i64, P(ctypes.c_int8)]
        L.orc_max_threads.restype = i32
        L.orc_set_threads.argtypes = [i32]
        _lib = L
    return _lib


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _i8(a):
    return np.ascontiguousarray(a, dtype=np.int8)


def max_threads() -> int:
    return int(lib().orc_max_threads())


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def sum_abs(W) -> float:
    W = _f32(W)
    return float(lib().orc_sum_abs(_p(W, ctypes.c_float), W.size))


def absmean_gamma(W) -> np.float32:
    W = _f32(W)
    N, K = W.shape
    return np.float32(lib().orc_absmean_gamma(_p(W, ctypes.c_float), N, K))


def ternary_codes(W, gamma, eps):
    W = _f32(W)
    N, K = W.shape
    out = np.empty((N, K), np.int8)
    lib().orc_ternary_codes(_p(W, ctypes.c_float), N, K, float(np.float32(gamma)),
                            float(np.float32(eps)), _p(out, ctypes.c_int8))
    return out


def quant_weights(W, eps):
    """quantise_weights_ternary: returns (codes int8 [N,K] in {-1,0,1}, γ fp32)."""
    W = _f32(W)
    N, K = W.shape
    out = np.empty((N, K), np.int8)
    g = lib().orc_quant_weights(_p(W, ctypes.c_float), N, K, float(np.float32(eps)),
                                _p(out, ctypes.c_int8))
    return out, np.float32(g)


def pack_ternary(Wq):
    Wq = _i8(Wq)
    N, K = Wq.shape
    assert K % 16 == 0
    out = np.empty((N, K // 4), np.uint8)
    lib().orc_pack_ternary(_p(Wq, ctypes.c_int8), N, K, _p(out, ctypes.c_uint8))
    return out


def unpack_ternary(packed, K):
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    assert packed.shape[1] * 4 == K
    out = np.empty((N, K), np.int8)
    bad = lib().orc_unpack_ternary(_p(packed, ctypes.c_uint8), N, K, _p(out, ctypes.c_int8))
    return out, int(bad)


def quant_acts(A, eps):
    """quantise_activations_8bit: returns (A_q int8 [M,K], γ_A fp32 [M])."""
    A = _f32(A)
    M, K = A.shape
    q = np.empty((M, K), np.int8)
    g = np.empty((M,), np.float32)
    lib().orc_quant_acts(_p(A, ctypes.c_float), M, K, float(np.float32(eps)),
                         _p(q, ctypes.c_int8), _p(g, ctypes.c_float))
    return q, g


def zero_gemm(Aq, Wq):
    Aq, Wq = _i8(Aq), _i8(Wq)
    M, K = Aq.shape
    N = Wq.shape[0]
    assert Wq.shape[1] == K
    acc = np.empty((M, N), np.int32)
    lib().orc_zero_gemm(_p(Aq, ctypes.c_int8), _p(Wq, ctypes.c_int8), M, N, K,
                        _p(acc, ctypes.c_int32))
    return acc


def lut_gemm(Aq, Wq):
    Aq, Wq = _i8(Aq), _i8(Wq)
    M, K = Aq.shape
    N = Wq.shape[0]
    assert Wq.shape[1] == K and K % 4 == 0
    acc = np.empty((M, N), np.int32)
    lib().orc_lut_gemm(_p(Aq, ctypes.c_int8), _p(Wq, ctypes.c_int8), M, N, K,
                       _p(acc, ctypes.c_int32))
    return acc


def dequant(acc, gammaA, gamma, relu2=False):
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    gA = _f32(gammaA)
    M, N = acc.shape
    Y = np.empty((M, N), np.float64)
    lib().orc_dequant(_p(acc, ctypes.c_int32), _p(gA, ctypes.c_float), float(np.float32(gamma)),
                      M, N, int(bool(relu2)), _p(Y, ctypes.c_double))
    return Y


def dequant_f32(acc, gammaA, gamma):
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    gA = _f32(gammaA)
    M, N = acc.shape
    H = np.empty((M, N), np.float32)
    lib().orc_dequant_f32(_p(acc, ctypes.c_int32), _p(gA, ctypes.c_float),
                          float(np.float32(gamma)), M, N, _p(H, ctypes.c_float))
    return H


def relu2_requant(acc_up, gammaA, g_up, eps):
    acc_up = np.ascontiguousarray(acc_up, dtype=np.int32)
    gA = _f32(gammaA)
    M, H = acc_up.shape
    q = np.empty((M, H), np.int8)
    g = np.empty((M,), np.float32)
    lib().orc_relu2_requant(_p(acc_up, ctypes.c_int32), _p(gA, ctypes.c_float),
                            float(np.float32(g_up)), M, H, float(np.float32(eps)),
                            _p(q, ctypes.c_int8), _p(g, ctypes.c_float))
    return q, g


def bitlinear(A, Wq, gamma, eps, relu2=False):
    """BitLinear forward from fp32 activations and ternary codes.
    Returns dict with Aq, gammaA, acc (int32) and Y (float64)."""
    Aq, gA = quant_acts(A, eps)
    acc = zero_gemm(Aq, Wq)
    Y = dequant(acc, gA, gamma, relu2)
    return {"Aq": Aq, "gammaA": gA, "acc": acc, "Y": Y}


def ffn_relu2(X, Wup, g_up, Wdown, g_down, eps):
    """Ternary FFN block: up BitLinear, ReLU², per-token requant, down BitLinear."""
    Xq, gX = quant_acts(X, eps)
    acc_up = zero_gemm(Xq, Wup)
    Rq, gR = relu2_requant(acc_up, gX, g_up, eps)
    acc_dn = zero_gemm(Rq, Wdown)
    Y = dequant(acc_dn, gR, g_down, False)
    return {"Xq": Xq, "gammaX": gX, "acc_up": acc_up, "Rq": Rq, "gammaR": gR,
            "acc_down": acc_dn, "Y": Y}


def ste_grad_input(dY, Wq, gamma):
    """STE backward, activation gradient: dA = dY·Ŵ with Ŵ = γ·W_q (float64)."""
    dY, Wq = _f32(dY), _i8(Wq)
    M, N = dY.shape
    K = Wq.shape[1]
    assert Wq.shape[0] == N
    dA = np.empty((M, K), np.float64)
    lib().orc_ste_grad_input(_p(dY, ctypes.c_float), M, N, _p(Wq, ctypes.c_int8), K,
                             float(np.float32(gamma)), _p(dA, ctypes.c_double))
    return dA


def ste_weight_mask(W, gamma, eps):
    """1 where -1 <= fp32(W / (γ+ε)) <= 1 (the clip was not active)."""
    W = _f32(W)
    N, K = W.shape
    mask = np.empty((N, K), np.uint8)
    lib().orc_ste_weight_mask(_p(W, ctypes.c_float), N, K, float(np.float32(gamma)),
                              float(np.float32(eps)), _p(mask, ctypes.c_uint8))
    return mask


def ste_grad_weight(dY, Aq, gammaA, W, gamma, eps):
    """STE backward, weight gradient: dW = mask ⊙ (dYᵀ·Â), Â = (γ_A/127)·A_q."""
    dY, Aq, gA, W = _f32(dY), _i8(Aq), _f32(gammaA), _f32(W)
    M, N = dY.shape
    K = Aq.shape[1]
    assert W.shape == (N, K) and gA.shape == (M,)
    dW = np.empty((N, K), np.float64)
    lib().orc_ste_grad_weight(_p(dY, ctypes.c_float), M, N, _p(Aq, ctypes.c_int8),
                              _p(gA, ctypes.c_float), K, _p(W, ctypes.c_float),
                              float(np.float32(gamma)), float(np.float32(eps)),
                              _p(dW, ctypes.c_double))
    return dW


def radix3_row_bytes(K: int) -> int:
    return int(lib().orc_radix3_row_bytes(K))


def pack_radix3(Wq):
    """Radix-3 storage: 5 ternary weights per byte (first most significant),
    byte = ceil(256·b/243); rows padded to 16 bytes."""
    Wq = _i8(Wq)
    N, K = Wq.shape
    out = np.empty((N, radix3_row_bytes(K)), np.uint8)
    lib().orc_pack_radix3(_p(Wq, ctypes.c_int8), N, K, _p(out, ctypes.c_uint8))
    return out


def unpack_radix3(packed, K):
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    assert packed.shape[1] == radix3_row_bytes(K)
    out = np.empty((N, K), np.int8)
    bad = lib().orc_unpack_radix3(_p(packed, ctypes.c_uint8), N, K, _p(out, ctypes.c_int8))
    return out, int(bad)
