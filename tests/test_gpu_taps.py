"""Bit-exact parity of the integers the path decides on its way, read out
through the taps of bl_linear_taps / bl_ffn_relu2_taps (C ABI).

"BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM", section "Por que
1,58 bits por peso ...", activation paragraph (AbsMax per token:
A_q = Clip(Round(A·127/(γ_A+ε)), -128, 127)); the FFN composes it with
ReLUSquared ("Arquitetura Hibrida Multimodal para bitnet.cpp", utils/): the
requantised r = max(h, 0)² of the dequantised up-projection.

Checked element by element against the oracle: the int8 tokens, γ_A and
Σ A_q that the fused decode-GEMV prologue makes (M ≤ 4; the first and the
last CTA, since every CTA quantises for itself), and in the FFN block the
quantised input X_q, the INT32 up-projection, the requantised R_q, γ_r and
Σ R_q, at M ∈ {1, 2, 4} (fused GEMV prologues) and {5, 32, 64, 512} (separate
kernels). Rounding-boundary exemptions are counted and printed in the
terminal summary; integers must otherwise be identical.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from parity_helpers import EPS, assert_acts_match, assert_close, assert_requant_match

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def bl():
    import ternary_weight_linear_absmax_b200 as m
    m.load()
    return m


def to_dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(DEV)


def _host(t):
    return {k: v.cpu().numpy() for k, v in t.items()}


@pytest.fixture(scope="module")
def decode_matrix():
    W = si.weights(6912, 2560, seed=0, dtype="bf16")
    codes, g = oracle.quant_weights(W.f32, EPS)
    return codes, g, to_dev(oracle.pack_ternary(codes)), to_dev(np.array([g], np.float32))


@pytest.mark.parametrize("cta", [0, -1])
@pytest.mark.parametrize("M", [1, 2, 4])
def test_gemv_prologue_tokens(bl, decode_matrix, M, cta):
    """Decode GEMV (K=2560, N=6912, bf16, 1 % ×20 outlier channels): the
    fused prologue's int8 tokens, γ_A and Σ A_q equal the oracle's."""
    codes, g, packed, gamma = decode_matrix
    A = si.activations(M, 2560, seed=40 + M, outliers=True, dtype="bf16")
    Y, t = bl.bl_linear_taps(A.torch(DEV), packed, gamma, EPS, cta=cta, pdl=True)
    t = _host(t)
    assert_acts_match(t["act_q"], t["act_gamma"], t["act_rowsum"], A.f32,
                      what=f"GEMV prologue M={M} cta={cta}")
    ref = oracle.bitlinear(A.f32, codes, g, EPS)["Y"]
    assert_close(Y.float().cpu().numpy(), ref, False)


@pytest.mark.parametrize("M,K,N,dt", [(3, 4096, 1000, "f32"), (1, 64, 300, "bf16"),
                                      (4, 11008, 512, "bf16")])
def test_gemv_prologue_tokens_shapes(bl, M, K, N, dt):
    W = si.weights(N, K, seed=7, dtype="bf16")
    codes, g = oracle.quant_weights(W.f32, EPS)
    A = si.activations(M, K, seed=8, outliers=True, dtype=dt)
    for cta in (0, -1):
        Y, t = bl.bl_linear_taps(A.torch(DEV), to_dev(oracle.pack_ternary(codes)),
                                 to_dev(np.array([g], np.float32)), EPS, cta=cta,
                                 out_dtype=torch.float32)
        t = _host(t)
        assert_acts_match(t["act_q"], t["act_gamma"], t["act_rowsum"], A.f32,
                          what=f"GEMV prologue {M}x{K}->{N} {dt} cta={cta}")
        ref = oracle.bitlinear(A.f32, codes, g, EPS)["Y"]
        assert_close(Y.cpu().numpy(), ref, True)


def test_linear_taps_separate_quantiser(bl):
    """Above the GEMV limit the taps are the quantiser kernel's outputs."""
    M, K, N = 40, 2560, 512
    W = si.weights(N, K, seed=3, dtype="bf16")
    codes, g = oracle.quant_weights(W.f32, EPS)
    A = si.activations(M, K, seed=4, outliers=True, dtype="bf16")
    Y, t = bl.bl_linear_taps(A.torch(DEV), to_dev(oracle.pack_ternary(codes)),
                             to_dev(np.array([g], np.float32)), EPS)
    t = _host(t)
    assert_acts_match(t["act_q"], t["act_gamma"], t["act_rowsum"], A.f32, what="linear M=40")


@pytest.fixture(scope="module")
def ffn_weights():
    K, H = 4096, 11008
    Wu = si.weights(H, K, seed=1, dtype="bf16")
    Wd = si.weights(K, H, seed=2, dtype="bf16")
    cu, gu = oracle.quant_weights(Wu.f32, EPS)
    cd, gd = oracle.quant_weights(Wd.f32, EPS)
    dev = (to_dev(oracle.pack_ternary(cu)), to_dev(np.array([gu], np.float32)),
           to_dev(oracle.pack_ternary(cd)), to_dev(np.array([gd], np.float32)))
    return cu, gu, cd, gd, dev


FFN_CASES = [(1, 0), (1, -1), (2, 0), (4, -1), (5, 0), (32, 0), (64, 0), (512, 0)]


@pytest.mark.parametrize("M,cta", FFN_CASES)
def test_ffn_intermediates(bl, ffn_weights, M, cta):
    """FFN block 4096 → 11008 → 4096 (bf16 in/out): X_q, γ_X, Σ X_q, the INT32
    up-projection, R_q, γ_r and Σ R_q bit-exact against the oracle; sampled
    tokens at M = 512 (the oracle recomputes those tokens from X alone)."""
    cu, gu, cd, gd, (pu, gu_d, pd, gd_d) = ffn_weights
    X = si.activations(M, 4096, seed=60 + M, outliers=True, dtype="bf16")
    Y, t = bl.bl_ffn_relu2_taps(X.torch(DEV), pu, gu_d, pd, gd_d, EPS, cta=cta)
    t = _host(t)
    tok = np.arange(M) if M <= 64 else np.array([0, 1, 255, 256, M - 1])
    Xq_ref, gX_ref = assert_acts_match(t["act_q"][tok], t["act_gamma"][tok],
                                       t["act_rowsum"][tok], X.f32[tok],
                                       what=f"FFN X_q M={M} cta={cta}")
    acc_ref = oracle.zero_gemm(Xq_ref, cu)
    np.testing.assert_array_equal(t["acc_up"][tok], acc_ref, err_msg="up-projection INT32")
    Rq_ref, gR_ref = assert_requant_match(t["req_q"][tok], t["req_gamma"][tok],
                                          t["req_rowsum"][tok], acc_ref, gX_ref, gu,
                                          what=f"FFN R_q M={M} cta={cta}")
    rows = np.concatenate([np.arange(0, 64), np.arange(4032, 4096)])
    ref = oracle.dequant(oracle.zero_gemm(Rq_ref, cd[rows]), gR_ref, gd)
    assert_close(Y.float().cpu().numpy()[np.ix_(tok, rows)], ref, False)
