"""BitNet b1.58 BitLinear forward on B200 (sm_100a): Python binding.

Thin marshalling layer over the C ABI of ``libbitlinear.so``
(``include/bitlinear.h``): each function has the name of the C entry point,
takes CUDA ``torch.Tensor`` arguments, allocates outputs and workspace with
torch, and passes raw device pointers plus the current CUDA stream. Every
computation happens in the library's CUDA kernels; there is no fallback.

Method: "BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM" (AbsMean
ternary weights, AbsMax per-token INT8 activations, INT32 add/subtract/skip
contraction, dequantisation by γ·γ_A/127) with the API names of the
utils/bit_layers.py library of "Arquitetura Hibrida Multimodal para
bitnet.cpp" (quantise_weights_ternary, quantise_activations_8bit, BitLinear,
ReLUSquared).
"""
from __future__ import annotations

import torch

from . import _lib
from ._lib import BL_BF16, BL_F32, BL_FLAG_PDL, BL_FLAG_RAW_I32, BitLinearError, BlTaps, check, load

__all__ = [
    "bl_quant_weights", "bl_quant_acts", "bl_zero_gemm", "bl_linear_q", "bl_linear",
    "bl_linear_noalloc", "bl_ffn_relu2", "bl_linear_taps", "bl_ffn_relu2_taps",
    "bl_ffn_tp_up", "bl_ffn_tp_down", "bl_dequant_i32", "bl_ste_grad_input", "bl_ste_grad_weight",
    "bl_pack_radix3", "bl_linear_radix3", "bl_pack_lut_index", "bl_linear_lut",
    "bl_probe_pdl_floor", "bl_check_device_error", "bl_selftest_wait_timeout",
    "bl_gemv_max_tokens", "bl_contraction_path", "workspace_bytes", "BitLinearError", "load", "BL_FLAG_PDL",
]

_DT = {torch.float32: BL_F32, torch.bfloat16: BL_BF16}


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dt(t: torch.Tensor, what: str) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"{what}: dtype {t.dtype} not supported (float32 or bfloat16)")
    return _DT[t.dtype]


def _cuda(t: torch.Tensor, what: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{what} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    return t


def _shape(t: torch.Tensor, shape: tuple, what: str) -> None:
    """The library takes plain pointers and sizes: every tensor handed to it
    must have exactly the shape the sizes describe, or a kernel would read or
    write past it."""
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{what} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _atleast(t: torch.Tensor, n: int, what: str) -> None:
    if t.numel() < n:
        raise ValueError(f"{what} must hold at least {n} elements, got {t.numel()}")


def _ws(nbytes: int, device) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def bl_gemv_max_tokens() -> int:
    return int(load().bl_gemv_max_tokens())


def bl_contraction_path(M: int, N: int, K: int, sms: int, split_ws_bytes: int = 0) -> int:
    """Kernel that contracts M int8 tokens with an N × K packed matrix on a
    device of `sms` SMs: 0 GEMV, 1 warp-level int8 MMA, 2 tensor-core tiles,
    3 tensor-core tiles with K split (-1: invalid sizes). Host logic only."""
    return int(load().bl_contraction_path(M, N, K, sms, split_ws_bytes))


def workspace_bytes(op: str, M: int, K: int, N: int) -> int:
    """Workspace size for 'quant_weights', 'zero_gemm', 'linear_q', 'linear'
    or 'ffn' (for 'ffn', N is the hidden size H)."""
    L = load()
    if op == "quant_weights":
        return int(L.bl_quant_weights_workspace_bytes(N, K))
    return int(getattr(L, f"bl_{op}_workspace_bytes" if op != "ffn" else "bl_ffn_workspace_bytes")(M, K, N))


def bl_quant_weights(W: torch.Tensor, eps: float = 1e-5, *, out=None, gamma=None,
                     workspace=None, stream=None):
    """quantise_weights_ternary: W [N, K] fp32/bf16 → (packed uint8 [N, K/4], γ fp32 [1])."""
    _cuda(W, "W")
    N, K = W.shape
    if out is None:
        out = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    _cuda(out, "out")
    _shape(out, (N, K // 4), "out")
    if gamma is None:
        gamma = torch.empty((1,), dtype=torch.float32, device=W.device)
    _cuda(gamma, "gamma")
    _atleast(gamma, 1, "gamma")
    L = load()
    if workspace is None:
        workspace = _ws(int(L.bl_quant_weights_workspace_bytes(N, K)), W.device)
    else:
        _cuda(workspace, "workspace")
    check(L.bl_quant_weights(W.data_ptr(), _dt(W, "W"), N, K, float(eps), out.data_ptr(),
                             gamma.data_ptr(), _ptr(workspace), _nbytes(workspace),
                             _stream(stream)), "bl_quant_weights")
    return out, gamma


def bl_quant_acts(A: torch.Tensor, eps: float = 1e-5, *, rowsum: bool = True, stream=None):
    """quantise_activations_8bit: A [M, K] → (A_q int8 [M,K], γ_A fp32 [M], Σ A_q int32 [M] or None)."""
    _cuda(A, "A")
    M, K = A.shape
    Aq = torch.empty((M, K), dtype=torch.int8, device=A.device)
    gA = torch.empty((M,), dtype=torch.float32, device=A.device)
    rs = torch.empty((M,), dtype=torch.int32, device=A.device) if rowsum else None
    check(load().bl_quant_acts(A.data_ptr(), _dt(A, "A"), M, K, float(eps), Aq.data_ptr(),
                               gA.data_ptr(), _ptr(rs), _stream(stream)), "bl_quant_acts")
    return Aq, gA, rs


def bl_zero_gemm(A_q: torch.Tensor, W_packed: torch.Tensor, *, stream=None):
    """INT32 contraction acc[M, N] = A_q · W_qᵀ."""
    _cuda(A_q, "A_q")
    _cuda(W_packed, "W_packed")
    M, K = A_q.shape
    N = W_packed.shape[0]
    if W_packed.shape[1] * 4 != K:
        raise ValueError("W_packed must be [N, K/4]")
    acc = torch.empty((M, N), dtype=torch.int32, device=A_q.device)
    L = load()
    ws = _ws(int(L.bl_zero_gemm_workspace_bytes(M, K, N)), A_q.device)
    check(L.bl_zero_gemm(A_q.data_ptr(), M, K, W_packed.data_ptr(), N, acc.data_ptr(), _ptr(ws),
                         _nbytes(ws), _stream(stream)), "bl_zero_gemm")
    return acc


def bl_linear_q(A_q, gamma_A, W_packed, gamma, *, rowsum=None, relu2=False,
                out_dtype=torch.bfloat16, out=None, pdl=False, stream=None):
    """Y = (A_q·W_qᵀ)·(γ_A·γ)/127 (ReLU² optional) from int8 tokens.
    pdl: BL_FLAG_PDL (the kernel before this call does not write W_packed)."""
    for t, n in ((A_q, "A_q"), (gamma_A, "gamma_A"), (W_packed, "W_packed"), (gamma, "gamma")):
        _cuda(t, n)
    M, K = A_q.shape
    N = W_packed.shape[0]
    _shape(W_packed, (N, K // 4), "W_packed")
    if K % 4:
        raise ValueError("K must be a multiple of 4")
    _atleast(gamma_A, M, "gamma_A")
    _atleast(gamma, 1, "gamma")
    if rowsum is not None:
        _cuda(rowsum, "rowsum")
        _atleast(rowsum, M, "rowsum")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=A_q.device)
    _cuda(out, "out")
    _shape(out, (M, N), "out")
    L = load()
    ws = None if rowsum is not None else _ws(int(L.bl_linear_q_workspace_bytes(M, K, N)), A_q.device)
    check(L.bl_linear_q_ex(A_q.data_ptr(), gamma_A.data_ptr(), _ptr(rowsum), M, K,
                           W_packed.data_ptr(), gamma.data_ptr(), N, int(bool(relu2)),
                           out.data_ptr(), _dt(out, "out"), _ptr(ws), _nbytes(ws),
                           BL_FLAG_PDL if pdl else 0, _stream(stream)), "bl_linear_q")
    return out


def bl_linear(A, W_packed, gamma, eps: float = 1e-5, *, relu2=False, out_dtype=torch.bfloat16,
              out=None, workspace=None, pdl=False, stream=None):
    """BitLinear forward: Y [M, N] = dequant(quant(A) · W_qᵀ), ReLU² optional."""
    _cuda(A, "A")
    _cuda(W_packed, "W_packed")
    _cuda(gamma, "gamma")
    M, K = A.shape
    N = W_packed.shape[0]
    _shape(W_packed, (N, K // 4), "W_packed")
    _atleast(gamma, 1, "gamma")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=A.device)
    _cuda(out, "out")
    _shape(out, (M, N), "out")
    L = load()
    if workspace is None:
        workspace = _ws(int(L.bl_linear_workspace_bytes(M, K, N)), A.device)
    else:
        _cuda(workspace, "workspace")
    check(L.bl_linear_ex(A.data_ptr(), _dt(A, "A"), M, K, W_packed.data_ptr(), gamma.data_ptr(),
                         N, float(eps), int(bool(relu2)), out.data_ptr(), _dt(out, "out"),
                         _ptr(workspace), _nbytes(workspace), BL_FLAG_PDL if pdl else 0,
                         _stream(stream)), "bl_linear")
    return out


def bl_linear_noalloc(A, W_packed, gamma, eps: float = 1e-5, *, relu2=False,
                      out_dtype=torch.bfloat16, out=None, stream=None):
    """BitLinear forward that allocates no device memory inside the library
    (for callers without an allocator): the scratch comes from a fixed 4 MiB
    array in the library; larger problems raise BL_ERR_WORKSPACE. Only the
    output (when ``out`` is None) is allocated here, by torch."""
    _cuda(A, "A")
    _cuda(W_packed, "W_packed")
    _cuda(gamma, "gamma")
    M, K = A.shape
    N = W_packed.shape[0]
    _shape(W_packed, (N, K // 4), "W_packed")
    _atleast(gamma, 1, "gamma")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=A.device)
    _cuda(out, "out")
    _shape(out, (M, N), "out")
    check(load().bl_linear_noalloc(A.data_ptr(), _dt(A, "A"), M, K, W_packed.data_ptr(),
                                   gamma.data_ptr(), N, float(eps), int(bool(relu2)),
                                   out.data_ptr(), _dt(out, "out"), _stream(stream)),
          "bl_linear_noalloc")
    return out


def bl_ffn_relu2(X, W_up, gamma_up, W_down, gamma_down, eps: float = 1e-5, *,
                 out_dtype=torch.bfloat16, out=None, workspace=None, pdl=False, stream=None):
    """Ternary FFN block: BitLinear up (K→H), ReLU², per-token requant, BitLinear down (H→K)."""
    for t, n in ((X, "X"), (W_up, "W_up"), (gamma_up, "gamma_up"), (W_down, "W_down"),
                 (gamma_down, "gamma_down")):
        _cuda(t, n)
    M, K = X.shape
    H = W_up.shape[0]
    _shape(W_up, (H, K // 4), "W_up")
    _shape(W_down, (K, H // 4), "W_down")
    _atleast(gamma_up, 1, "gamma_up")
    _atleast(gamma_down, 1, "gamma_down")
    if out is None:
        out = torch.empty((M, K), dtype=out_dtype, device=X.device)
    _cuda(out, "out")
    _shape(out, (M, K), "out")
    L = load()
    if workspace is None:
        workspace = _ws(int(L.bl_ffn_workspace_bytes(M, K, H)), X.device)
    else:
        _cuda(workspace, "workspace")
    check(L.bl_ffn_relu2_ex(X.data_ptr(), _dt(X, "X"), M, K, H, W_up.data_ptr(), gamma_up.data_ptr(),
                            W_down.data_ptr(), gamma_down.data_ptr(), float(eps), out.data_ptr(),
                            _dt(out, "out"), _ptr(workspace), _nbytes(workspace),
                            BL_FLAG_PDL if pdl else 0, _stream(stream)), "bl_ffn_relu2")
    return out


def _taps(M, K, H, device, ffn: bool, cta: int):
    """Allocate tap buffers (torch) and the matching bl_taps structure."""
    t = {"act_q": torch.empty((M, K), dtype=torch.int8, device=device),
         "act_gamma": torch.empty((M,), dtype=torch.float32, device=device),
         "act_rowsum": torch.empty((M,), dtype=torch.int32, device=device)}
    if ffn:
        t.update({"acc_up": torch.empty((M, H), dtype=torch.int32, device=device),
                  "req_q": torch.empty((M, H), dtype=torch.int8, device=device),
                  "req_gamma": torch.empty((M,), dtype=torch.float32, device=device),
                  "req_rowsum": torch.empty((M,), dtype=torch.int32, device=device)})
    s = BlTaps(**{k: v.data_ptr() for k, v in t.items()}, cta=int(cta), reserved=0)
    return t, s


def bl_linear_taps(A, W_packed, gamma, eps: float = 1e-5, *, relu2=False,
                   out_dtype=torch.bfloat16, pdl=False, cta: int = 0, stream=None):
    """bl_linear that also returns the int8 tokens, γ_A and Σ A_q the
    contraction used (for the fused GEMV path: those of CTA ``cta``; -1 =
    the last CTA). Returns (Y, taps dict)."""
    _cuda(A, "A")
    _cuda(W_packed, "W_packed")
    _cuda(gamma, "gamma")
    M, K = A.shape
    N = W_packed.shape[0]
    _shape(W_packed, (N, K // 4), "W_packed")
    _atleast(gamma, 1, "gamma")
    out = torch.empty((M, N), dtype=out_dtype, device=A.device)
    L = load()
    ws = _ws(int(L.bl_linear_workspace_bytes(M, K, N)), A.device)
    taps, s = _taps(M, K, 0, A.device, False, cta)
    check(L.bl_linear_taps(A.data_ptr(), _dt(A, "A"), M, K, W_packed.data_ptr(), gamma.data_ptr(),
                           N, float(eps), int(bool(relu2)), out.data_ptr(), _dt(out, "out"),
                           _ptr(ws), _nbytes(ws), BL_FLAG_PDL if pdl else 0, s,
                           _stream(stream)), "bl_linear_taps")
    return out, taps


def bl_ffn_relu2_taps(X, W_up, gamma_up, W_down, gamma_down, eps: float = 1e-5, *,
                      out_dtype=torch.bfloat16, cta: int = 0, stream=None):
    """bl_ffn_relu2 that also returns X_q, γ_X, Σ X_q, the up-projection
    accumulators, the requantised ReLU² tokens R_q, γ_r and Σ R_q.
    Returns (Y, taps dict)."""
    for t, n in ((X, "X"), (W_up, "W_up"), (gamma_up, "gamma_up"), (W_down, "W_down"),
                 (gamma_down, "gamma_down")):
        _cuda(t, n)
    M, K = X.shape
    H = W_up.shape[0]
    _shape(W_up, (H, K // 4), "W_up")
    _shape(W_down, (K, H // 4), "W_down")
    out = torch.empty((M, K), dtype=out_dtype, device=X.device)
    L = load()
    ws = _ws(int(L.bl_ffn_workspace_bytes(M, K, H)), X.device)
    taps, s = _taps(M, K, H, X.device, True, cta)
    check(L.bl_ffn_relu2_taps(X.data_ptr(), _dt(X, "X"), M, K, H, W_up.data_ptr(),
                              gamma_up.data_ptr(), W_down.data_ptr(), gamma_down.data_ptr(),
                              float(eps), out.data_ptr(), _dt(out, "out"), _ptr(ws), _nbytes(ws),
                              s, _stream(stream)), "bl_ffn_relu2_taps")
    return out, taps


def bl_ffn_tp_up(X, W_up_r, gamma_up, eps: float = 1e-5, *, stream=None):
    """Tensor-parallel FFN, step 1 on this rank's shard of H: returns
    (acc_up int32 [M, H_r], γ_X fp32 [M], rmax fp32 [M] = shard max of r)."""
    _cuda(X, "X")
    _cuda(W_up_r, "W_up_r")
    _cuda(gamma_up, "gamma_up")
    M, K = X.shape
    H_r = W_up_r.shape[0]
    if W_up_r.shape[1] * 4 != K:
        raise ValueError("W_up_r must be [H_r, K/4]")
    acc = torch.empty((M, H_r), dtype=torch.int32, device=X.device)
    gX = torch.empty((M,), dtype=torch.float32, device=X.device)
    rmax = torch.empty((M,), dtype=torch.float32, device=X.device)
    L = load()
    ws = _ws(int(L.bl_ffn_tp_up_workspace_bytes(M, K)), X.device)
    check(L.bl_ffn_tp_up(X.data_ptr(), _dt(X, "X"), M, K, H_r, W_up_r.data_ptr(),
                         gamma_up.data_ptr(), float(eps), acc.data_ptr(), gX.data_ptr(),
                         rmax.data_ptr(), _ptr(ws), _nbytes(ws), _stream(stream)), "bl_ffn_tp_up")
    return acc, gX, rmax


def bl_ffn_tp_down(acc_up, gamma_x, gamma_up, gamma_r, W_down_r, eps: float = 1e-5, *,
                   stream=None):
    """Tensor-parallel FFN, step 3: requantise this shard with the all-ranks
    γ_r and return its partial down-projection (int32 [M, K_out])."""
    for t, n in ((acc_up, "acc_up"), (gamma_x, "gamma_x"), (gamma_up, "gamma_up"),
                 (gamma_r, "gamma_r"), (W_down_r, "W_down_r")):
        _cuda(t, n)
    M, H_r = acc_up.shape
    K_out = W_down_r.shape[0]
    if W_down_r.shape[1] * 4 != H_r:
        raise ValueError("W_down_r must be [K_out, H_r/4]")
    out = torch.empty((M, K_out), dtype=torch.int32, device=acc_up.device)
    L = load()
    ws = _ws(int(L.bl_ffn_tp_down_workspace_bytes(M, H_r)), acc_up.device)
    check(L.bl_ffn_tp_down(acc_up.data_ptr(), gamma_x.data_ptr(), gamma_up.data_ptr(),
                           gamma_r.data_ptr(), M, H_r, W_down_r.data_ptr(), K_out, float(eps),
                           out.data_ptr(), _ptr(ws), _nbytes(ws), _stream(stream)), "bl_ffn_tp_down")
    return out


def bl_dequant_i32(acc, gamma_A, gamma, *, relu2=False, out_dtype=torch.bfloat16, stream=None):
    """Y = acc · ((γ_A·γ)/127) (ReLU² optional) from INT32 accumulators."""
    for t, n in ((acc, "acc"), (gamma_A, "gamma_A"), (gamma, "gamma")):
        _cuda(t, n)
    M, N = acc.shape
    out = torch.empty((M, N), dtype=out_dtype, device=acc.device)
    check(load().bl_dequant_i32(acc.data_ptr(), gamma_A.data_ptr(), gamma.data_ptr(), M, N,
                                int(bool(relu2)), out.data_ptr(), _dt(out, "out"),
                                _stream(stream)), "bl_dequant_i32")
    return out


def bl_pack_radix3(W_packed, K: int, *, out=None, stream=None):
    """2-bit packed [N, K/4] → radix-3 storage [N, row_bytes] (5 weights/byte)."""
    _cuda(W_packed, "W_packed")
    N = W_packed.shape[0]
    _shape(W_packed, (N, K // 4), "W_packed")
    L = load()
    rb = int(L.bl_radix3_row_bytes(K))
    if out is None:
        out = torch.empty((N, rb), dtype=torch.uint8, device=W_packed.device)
    _cuda(out, "out")
    _shape(out, (N, rb), "out")
    check(L.bl_pack_radix3(W_packed.data_ptr(), N, K, out.data_ptr(), _stream(stream)),
          "bl_pack_radix3")
    return out


def bl_linear_radix3(A, W_r3, gamma, eps: float = 1e-5, *, relu2=False, out_dtype=torch.bfloat16,
                     raw=False, out=None, pdl=False, stream=None):
    """BitLinear for ≤ 4 tokens on radix-3 weights (raw=True: INT32 accumulators)."""
    _cuda(A, "A")
    _cuda(W_r3, "W_r3")
    _cuda(gamma, "gamma")
    M, K = A.shape
    N = W_r3.shape[0]
    _shape(W_r3, (N, int(load().bl_radix3_row_bytes(K))), "W_r3")
    _atleast(gamma, 1, "gamma")
    if out is None:
        out = torch.empty((M, N), dtype=torch.int32 if raw else out_dtype, device=A.device)
    _cuda(out, "out")
    _shape(out, (M, N), "out")
    if raw and out.dtype != torch.int32:
        raise TypeError("out must be int32 when raw=True")
    flags = (BL_FLAG_PDL if pdl else 0) | (BL_FLAG_RAW_I32 if raw else 0)
    ydt = BL_F32 if raw else _dt(out, "out")
    check(load().bl_linear_radix3(A.data_ptr(), _dt(A, "A"), M, K, W_r3.data_ptr(), gamma.data_ptr(),
                                  N, float(eps), int(bool(relu2)), out.data_ptr(), ydt, flags,
                                  _stream(stream)), "bl_linear_radix3")
    return out


def bl_pack_lut_index(W_packed, *, out=None, stream=None):
    """2-bit packed [N, K/4] → lookup-table index bytes [N, K/4]."""
    _cuda(W_packed, "W_packed")
    N, Kq = W_packed.shape
    if out is None:
        out = torch.empty((N, Kq), dtype=torch.uint8, device=W_packed.device)
    _cuda(out, "out")
    _shape(out, (N, Kq), "out")
    check(load().bl_pack_lut_index(W_packed.data_ptr(), N, 4 * Kq, out.data_ptr(), _stream(stream)),
          "bl_pack_lut_index")
    return out


def bl_linear_lut(A, W_idx, gamma, eps: float = 1e-5, *, out_dtype=torch.bfloat16, raw=False,
                  out=None, pdl=False, stream=None):
    """BitLinear for one token by table lookup (raw=True: INT32 accumulators)."""
    _cuda(A, "A")
    _cuda(W_idx, "W_idx")
    _cuda(gamma, "gamma")
    M, K = A.shape
    N = W_idx.shape[0]
    _shape(W_idx, (N, K // 4), "W_idx")
    _atleast(gamma, 1, "gamma")
    if out is None:
        out = torch.empty((M, N), dtype=torch.int32 if raw else out_dtype, device=A.device)
    _cuda(out, "out")
    _shape(out, (M, N), "out")
    if raw and out.dtype != torch.int32:
        raise TypeError("out must be int32 when raw=True")
    flags = (BL_FLAG_PDL if pdl else 0) | (BL_FLAG_RAW_I32 if raw else 0)
    check(load().bl_linear_lut(A.data_ptr(), _dt(A, "A"), M, K, W_idx.data_ptr(), gamma.data_ptr(),
                               N, float(eps), out.data_ptr(), BL_F32 if raw else _dt(out, "out"),
                               flags, _stream(stream)), "bl_linear_lut")
    return out


def bl_ste_grad_input(dY, W_packed, gamma, *, stream=None):
    """STE backward, activation gradient dA [M, K] = γ·(dY·W_q) (fp32)."""
    _cuda(dY, "dY")
    _cuda(W_packed, "W_packed")
    _cuda(gamma, "gamma")
    M, N = dY.shape
    if W_packed.shape[0] != N:
        raise ValueError("W_packed must be [N, K/4] with N = dY.shape[1]")
    K = W_packed.shape[1] * 4
    dA = torch.empty((M, K), dtype=torch.float32, device=dY.device)
    L = load()
    ws = _ws(int(L.bl_ste_grad_input_workspace_bytes(M, N, K)), dY.device)
    check(L.bl_ste_grad_input(dY.data_ptr(), _dt(dY, "dY"), M, N, W_packed.data_ptr(),
                              gamma.data_ptr(), K, dA.data_ptr(), _ptr(ws), _nbytes(ws),
                              _stream(stream)), "bl_ste_grad_input")
    return dA


def bl_ste_grad_weight(dY, A_q, gamma_A, W, gamma, eps: float = 1e-5, *, stream=None):
    """STE backward, weight gradient dW [N, K] = mask ⊙ (dYᵀ·Â) (fp32); W are
    the latent weights [N, K] whose clip range makes the mask."""
    for t, n in ((dY, "dY"), (A_q, "A_q"), (gamma_A, "gamma_A"), (W, "W"), (gamma, "gamma")):
        _cuda(t, n)
    M, N = dY.shape
    K = A_q.shape[1]
    if A_q.shape[0] != M or tuple(W.shape) != (N, K):
        raise ValueError("A_q must be [M, K] and W [N, K]")
    dW = torch.empty((N, K), dtype=torch.float32, device=dY.device)
    L = load()
    ws = _ws(int(L.bl_ste_grad_weight_workspace_bytes(M, N, K)), dY.device)
    check(L.bl_ste_grad_weight(dY.data_ptr(), _dt(dY, "dY"), M, N, A_q.data_ptr(),
                               gamma_A.data_ptr(), K, W.data_ptr(), _dt(W, "W"), gamma.data_ptr(),
                               float(eps), dW.data_ptr(), _ptr(ws), _nbytes(ws), _stream(stream)),
          "bl_ste_grad_weight")
    return dW


def bl_probe_pdl_floor(M: int, K: int, N: int, *, stream=None) -> None:
    """One empty kernel with the decode GEMV's launch shape for (M, K, N)."""
    check(load().bl_probe_pdl_floor(M, K, N, _stream(stream)), "bl_probe_pdl_floor")


def bl_check_device_error(stream=None) -> int:
    """Synchronise the stream; return the library status (0 = BL_OK)."""
    return int(load().bl_check_device_error(_stream(stream)))


def bl_selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    check(load().bl_selftest_wait_timeout(int(limit_ns), _stream(stream)),
          "bl_selftest_wait_timeout")
