"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol include/bitlinear.h declares, and rejects bad arguments on the
host with the documented status codes before touching a device."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "bitlinear.h")


@pytest.fixture(scope="module")
def lib():
    from ternary_weight_linear_absmax_b200 import _lib
    from ternary_weight_linear_absmax_b200 import build as b
    b.build()
    return _lib.load()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bl_[a-z0-9_]+)\s*\(", text)))


def test_header_symbols_exported(lib):
    from ternary_weight_linear_absmax_b200 import _lib
    syms = declared_symbols()
    assert len(syms) >= 15
    for s in syms:
        assert hasattr(lib, s), f"{s} declared in bitlinear.h but not exported"
    # the binding declares a signature for every exported entry point
    assert set(syms) == set(_lib.SIGNATURES)


def test_status_strings(lib):
    for code in range(9):
        s = lib.bl_status_string(code).decode()
        assert s.startswith("BL_")
    assert lib.bl_status_string(99).decode() == "BL_ERR_UNKNOWN"
    assert lib.bl_version() >= 100
    assert lib.bl_gemv_max_tokens() == 4


def test_contraction_path(lib):
    """Routing of a contraction (host logic, no device): GEMV up to 4 tokens,
    the warp-level kernel up to 32, tensor-core tiles above 64, and from 33 to
    64 tokens the tiles only when they (times their K ranges) fill at least
    half of the SMs."""
    P = lib.bl_contraction_path
    room = 1 << 40   # workspace with room for K-split partials
    assert P(1, 6912, 2560, 148, 0) == 0
    assert P(4, 6912, 2560, 148, room) == 0
    assert P(16, 11008, 4096, 148, room) == 1
    assert P(32, 11008, 4096, 148, room) == 1
    assert P(40, 11008, 4096, 148, room) == 2      # 86 tiles: 2·86 ≥ 148, unsplit
    assert P(64, 4096, 11008, 148, room) == 3      # 32 tiles × 4 K ranges
    assert P(64, 4096, 11008, 148, 0) == 1         # no room to split: 32 tiles
    assert P(48, 1500, 3200, 148, room) == 1       # 12 tiles × 3 ranges
    assert P(65, 200, 256, 148, 0) == 2
    assert P(2048, 4096, 4096, 148, room) == 2     # 256 tiles
    assert P(512, 4096, 11008, 148, room) == 3     # the FFN down-projection
    assert P(512, 4096, 11008, 148, 0) == 2
    assert P(40, 11008, 4096, 132, room) == 2      # another SM count
    assert P(0, 64, 64, 148, 0) == -1 and P(8, 64, 100, 148, 0) == -1
    # a few tokens whose rows do not fit the fused GEMV's shared memory
    assert P(1, 512, 37376, 148, 0) == 0 and P(1, 512, 37440, 148, 0) == 1
    assert P(4, 200, 18624, 148, 0) == 0 and P(4, 200, 18688, 148, 0) == 1
    assert lib.bl_linear_workspace_bytes(1, 37376, 512) == 0
    assert lib.bl_linear_workspace_bytes(1, 37440, 512) >= 37440 + 8
    assert lib.bl_zero_gemm_workspace_bytes(4, 18688, 200) >= 16


def test_workspace_sizes(lib):
    assert lib.bl_quant_weights_workspace_bytes(4096, 4096) >= 1024 * 8
    assert lib.bl_linear_workspace_bytes(1, 2560, 6912) == 0
    ws = lib.bl_linear_workspace_bytes(2048, 4096, 4096)
    assert ws >= 2048 * 4096 + 2 * 2048 * 4
    assert lib.bl_ffn_workspace_bytes(1, 4096, 11008) >= 11008 * 4 + 4
    assert lib.bl_ffn_workspace_bytes(512, 4096, 11008) >= 512 * 11008 * 5 + 512 * 4096
    assert lib.bl_zero_gemm_workspace_bytes(4, 512, 256) == 0


def _aligned_buf(n=4096):
    buf = ctypes.create_string_buffer(n + 64)
    addr = (ctypes.addressof(buf) + 15) & ~15
    return buf, addr


def test_argument_errors_on_host(lib):
    """Shape, eps, pointer, alignment, dtype and workspace errors are caught
    before any CUDA call (these run without a GPU)."""
    keep, p = _aligned_buf()
    BL_ERR_INVALID_ARG, BL_ERR_SHAPE, BL_ERR_ALIGN, BL_ERR_DTYPE, BL_ERR_WORKSPACE = 1, 2, 3, 4, 8
    # K not a multiple of 64
    assert lib.bl_quant_weights(p, 0, 16, 100, 1e-5, p, p, p, 8192, None) == BL_ERR_SHAPE
    assert lib.bl_quant_weights(p, 0, 16, 0, 1e-5, p, p, p, 8192, None) == BL_ERR_SHAPE
    assert lib.bl_quant_weights(p, 0, -1, 64, 1e-5, p, p, p, 8192, None) == BL_ERR_SHAPE
    # eps must be > 0 and finite
    assert lib.bl_quant_weights(p, 0, 16, 64, 0.0, p, p, p, 8192, None) == BL_ERR_INVALID_ARG
    assert lib.bl_quant_weights(p, 0, 16, 64, float("nan"), p, p, p, 8192, None) == BL_ERR_INVALID_ARG
    # dtype
    assert lib.bl_quant_weights(p, 7, 16, 64, 1e-5, p, p, p, 8192, None) == BL_ERR_DTYPE
    # null and misaligned pointers
    assert lib.bl_quant_weights(None, 0, 16, 64, 1e-5, p, p, p, 8192, None) == BL_ERR_INVALID_ARG
    assert lib.bl_quant_weights(p + 4, 0, 16, 64, 1e-5, p, p, p, 8192, None) == BL_ERR_ALIGN
    # workspace
    assert lib.bl_quant_weights(p, 0, 16, 64, 1e-5, p, p, None, 0, None) == BL_ERR_WORKSPACE
    assert lib.bl_quant_weights(p, 0, 16, 64, 1e-5, p, p, p, 16, None) == BL_ERR_WORKSPACE
    # linear: workspace required above the GEMV token limit
    assert lib.bl_linear(p, 1, 64, 512, p, p, 256, 1e-5, 0, p, 1, None, 0, None) == BL_ERR_WORKSPACE
    assert lib.bl_linear(p, 1, 4, 500, p, p, 256, 1e-5, 0, p, 1, None, 0, None) == BL_ERR_SHAPE
    assert lib.bl_linear_ex(p, 1, 4, 512, p, p, 256, 1e-5, 0, p, 1, None, 0, 8, None) == BL_ERR_INVALID_ARG
    # FFN hidden size must be a multiple of 64
    assert lib.bl_ffn_relu2(p, 1, 1, 512, 100, p, p, p, p, 1e-5, p, 1, p, 1 << 20, None) == BL_ERR_SHAPE
    # empty problems are no-ops
    assert lib.bl_linear(p, 1, 0, 512, p, p, 256, 1e-5, 0, p, 1, None, 0, None) == 0
    assert lib.bl_quant_acts(p, 1, 0, 512, 1e-5, p, p, None, None) == 0
    assert lib.bl_selftest_wait_timeout(10, None) == BL_ERR_INVALID_ARG


def test_k_bound_and_taps_checked_on_host(lib):
    """K (and H) above 2^22 is refused (INT32 sums could no longer be exact);
    tap structures are validated before any launch."""
    from ternary_weight_linear_absmax_b200._lib import BlTaps
    keep, p = _aligned_buf()
    BL_ERR_INVALID_ARG, BL_ERR_SHAPE, BL_ERR_ALIGN = 1, 2, 3
    kmax = 1 << 22
    assert lib.bl_quant_acts(p, 1, 1, kmax + 64, 1e-5, p, p, None, None) == BL_ERR_SHAPE
    assert lib.bl_ffn_relu2(p, 1, 1, 512, kmax + 64, p, p, p, p, 1e-5, p, 1, p, 1 << 20,
                            None) == BL_ERR_SHAPE
    # K = 2^22 itself passes the shape check (M = 0: no-op, no device touched)
    assert lib.bl_quant_acts(p, 1, 0, kmax, 1e-5, p, p, None, None) == 0
    bad = BlTaps(reserved=1)
    assert lib.bl_linear_taps(p, 1, 4, 512, p, p, 256, 1e-5, 0, p, 1, None, 0, 0, bad,
                              None) == BL_ERR_INVALID_ARG
    ffn_only = BlTaps(acc_up=p)
    assert lib.bl_linear_taps(p, 1, 4, 512, p, p, 256, 1e-5, 0, p, 1, None, 0, 0, ffn_only,
                              None) == BL_ERR_INVALID_ARG
    misaligned = BlTaps(act_q=p + 8, act_gamma=p, act_rowsum=p)
    assert lib.bl_linear_taps(p, 1, 4, 512, p, p, 256, 1e-5, 0, p, 1, None, 0, 0, misaligned,
                              None) == BL_ERR_ALIGN
    assert lib.bl_ffn_relu2_taps(p, 1, 1, 512, 640, p, p, p, p, 1e-5, p, 1, p, 1 << 20,
                                 misaligned, None) == BL_ERR_ALIGN


def test_radix3_host_checks(lib):
    keep, p = _aligned_buf()
    BL_ERR_INVALID_ARG, BL_ERR_SHAPE = 1, 2
    assert lib.bl_radix3_row_bytes(2560) == 512
    assert lib.bl_radix3_row_bytes(4096) == 832
    # more than 4 tokens, bad flags, bad K: refused before any launch
    assert lib.bl_linear_radix3(p, 1, 5, 512, p, p, 64, 1e-5, 0, p, 1, 0, None) == BL_ERR_SHAPE
    assert lib.bl_linear_radix3(p, 1, 1, 512, p, p, 64, 1e-5, 0, p, 1, 4, None) == BL_ERR_INVALID_ARG
    assert lib.bl_linear_radix3(p, 1, 1, 500, p, p, 64, 1e-5, 0, p, 1, 0, None) == BL_ERR_SHAPE
    assert lib.bl_pack_radix3(p, 8, 100, p, None) == BL_ERR_SHAPE


def test_lut_host_checks(lib):
    keep, p = _aligned_buf()
    BL_ERR_INVALID_ARG, BL_ERR_SHAPE = 1, 2
    assert lib.bl_linear_lut(p, 1, 2, 512, p, p, 64, 1e-5, p, 1, 0, None) == BL_ERR_SHAPE
    assert lib.bl_linear_lut(p, 1, 1, 512, p, p, 64, 1e-5, p, 1, 8, None) == BL_ERR_INVALID_ARG
    assert lib.bl_pack_lut_index(p, 8, 100, p, None) == BL_ERR_SHAPE


def test_binding_shape_checks():
    """The library takes plain pointers and sizes, so the binding refuses
    tensors whose shapes do not match the sizes it passes (a packed matrix
    with a different K would be read past its end)."""
    import torch
    from ternary_weight_linear_absmax_b200 import _atleast, _shape
    _shape(torch.empty(8, 16), (8, 16), "W_packed")
    with pytest.raises(ValueError, match="W_packed must have shape"):
        _shape(torch.empty(8, 12), (8, 16), "W_packed")
    with pytest.raises(ValueError, match="out must have shape"):
        _shape(torch.empty(4, 8), (8, 4), "out")
    _atleast(torch.empty(3), 3, "gamma_A")
    with pytest.raises(ValueError, match="gamma_A must hold at least 4"):
        _atleast(torch.empty(3), 4, "gamma_A")
