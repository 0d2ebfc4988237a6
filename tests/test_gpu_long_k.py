"""Few tokens (M ≤ 4) with rows too long for the fused GEMV, through the C ABI
against the oracle.

"BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM", sections on
BitLinear and Zero-GEMM: the same contraction and scales at any K. The fused
GEMV holds a weight row and the M token rows in one CTA's shared memory (K up
to 37,376 at 1 token and 18,624 at 4); longer rows take the activation
quantiser and the warp-level kernel, and the workspaces grow to match. Same
bars as the other parity tests: INT32 bit-exact, outputs within the fp32 /
bf16 tolerances.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from parity_helpers import EPS, assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def bl():
    import ternary_weight_linear_absmax_b200 as m
    m.load()
    return m


def to_dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(DEV)


def _codes(N, K, seed):
    u = si.uniform(seed, N * K).reshape(N, K)
    return (np.floor(u * 3.0).astype(np.int8) - 1)


@pytest.mark.parametrize("M,K,N", [(1, 37440, 300), (2, 28160, 257), (4, 18688, 130),
                                   (4, 40000 // 64 * 64, 64)])
def test_zero_gemm_long_rows(bl, M, K, N):
    assert bl.bl_contraction_path(M, N, K, 148, 0) == 1
    u = si.uniform(M * 7 + K, M * K).reshape(M, K)
    Aq = (-127 + np.floor(u * 255)).astype(np.int8)
    codes = _codes(N, K, seed=N + K)
    acc = bl.bl_zero_gemm(to_dev(Aq), to_dev(oracle.pack_ternary(codes))).cpu().numpy()
    np.testing.assert_array_equal(acc, oracle.zero_gemm(Aq, codes))


@pytest.mark.parametrize("M,K,N,dt", [(1, 37376, 512, "bf16"), (1, 37440, 512, "bf16"),
                                      (2, 28672, 384, "f32"), (4, 18688, 200, "bf16")])
def test_linear_long_rows(bl, M, K, N, dt):
    """Both sides of the limit at 1 token (37,376 takes the GEMV, 37,440 does
    not) and past it at 2 and 4 tokens; bl_linear_q too."""
    W = si.weights(N, K, seed=K + 1, dtype="bf16")
    codes, g = oracle.quant_weights(W.f32, EPS)
    A = si.activations(M, K, seed=K + 2, outliers=True, dtype=dt)
    packed = to_dev(oracle.pack_ternary(codes))
    gd = to_dev(np.array([g], np.float32))
    out = torch.float32 if dt == "f32" else torch.bfloat16
    Y = bl.bl_linear(A.torch(DEV), packed, gd, EPS, out_dtype=out).float().cpu().numpy()
    ref = oracle.bitlinear(A.f32, codes, g, EPS)
    assert_close(Y, ref["Y"], dt == "f32")
    Aq, gA = oracle.quant_acts(A.f32, EPS)
    Yq = bl.bl_linear_q(to_dev(Aq), to_dev(gA), packed, gd, out_dtype=torch.float32).cpu().numpy()
    assert_close(Yq, oracle.dequant(oracle.zero_gemm(Aq, codes), gA, g), True)


@pytest.mark.parametrize("M", [2, 4])
def test_ffn_long_hidden(bl, M):
    """A hidden size of 28,672 (a 70B-class model's FFN): the down-projection's
    rows are too long for the GEMV at 2 and 4 tokens, so the block takes the
    separate quantiser, requantiser and warp-level kernels."""
    K, H = 1024, 28672
    cu, gu = oracle.quant_weights(si.weights(H, K, seed=61, dtype="bf16").f32, EPS)
    cd, gd = oracle.quant_weights(si.weights(K, H, seed=62, dtype="bf16").f32, EPS)
    X = si.activations(M, K, seed=63 + M, outliers=True, dtype="bf16")
    Y = bl.bl_ffn_relu2(X.torch(DEV), to_dev(oracle.pack_ternary(cu)), to_dev(np.array([gu], np.float32)),
                        to_dev(oracle.pack_ternary(cd)), to_dev(np.array([gd], np.float32)),
                        EPS).float().cpu().numpy()
    ref = oracle.ffn_relu2(X.f32, cu, gu, cd, gd, EPS)
    assert_close(Y, ref["Y"], False)
    # the tensor-parallel steps on one shard holding all 28,672 hidden rows
    pu, pd = to_dev(oracle.pack_ternary(cu)), to_dev(oracle.pack_ternary(cd))
    gu_d = to_dev(np.array([gu], np.float32))
    acc_up, gX, rmax = bl.bl_ffn_tp_up(X.torch(DEV), pu, gu_d, EPS)
    acc_down = bl.bl_ffn_tp_down(acc_up, gX, gu_d, rmax, pd, EPS)
    np.testing.assert_array_equal(acc_up.cpu().numpy(), ref["acc_up"])
    np.testing.assert_array_equal(rmax.cpu().numpy(), ref["gammaR"])
    np.testing.assert_array_equal(acc_down.cpu().numpy(), ref["acc_down"])
