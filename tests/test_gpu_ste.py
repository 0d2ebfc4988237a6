"""STE backward (bl_ste_grad_input, bl_ste_grad_weight) through the C ABI
against the oracle.

"BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM", STE paragraph:
dA = dY·Ŵ and dW = mask ⊙ dYᵀ·Â (mask: the forward's clip range).

Tolerance, from the arithmetic: both contractions run on the tensor cores
with bf16 operands and fp32 accumulation. W_q is exact in bf16; dY (when
fp32) and Â are rounded to bf16 once (relative 2^-9 each), products are
exact in fp32, and fp32 accumulation over L ≤ 2^14 terms adds at most
L·2^-24 ≤ 2^-10 relative to the sum of magnitudes. So every output must lie
within 2^-7 · S of the oracle's float64 value, where S is the sum of
|term| magnitudes (computed in float64 from the oracle's inputs). Where
the mask is 0 the gradient must be exactly 0.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si

pytestmark = pytest.mark.gpu
EPS = 1e-5
DEV = "cuda"


@pytest.fixture(scope="module")
def bl():
    import ternary_weight_linear_absmax_b200 as m
    m.load()
    return m


def to_dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(DEV)


def _problem(M, N, K, seed, dy_dtype):
    W = si.weights(N, K, seed=seed, dtype="bf16")
    codes, g = oracle.quant_weights(W.f32, EPS)
    A = si.activations(M, K, seed=seed + 1, outliers=True, dtype="bf16")
    Aq, gA = oracle.quant_acts(A.f32, EPS)
    dY = si.activations(M, N, seed=seed + 2, dtype=dy_dtype)
    return W, codes, g, Aq, gA, dY


CASES = [(4, 256, 512, "f32"), (130, 200, 320, "bf16"), (256, 1024, 768, "bf16"),
         (37, 512, 4096, "f32"), (512, 2048, 1024, "bf16"),
         # more output tiles than SMs (two CTAs per SM): dW of (64, 4096, 1536), dA of (2560, 128, 2048)
         (64, 4096, 1536, "bf16"), (2560, 128, 2048, "bf16")]


@pytest.mark.parametrize("M,N,K,dt", CASES)
def test_ste_grad_input(bl, M, N, K, dt):
    W, codes, g, Aq, gA, dY = _problem(M, N, K, seed=M + N, dy_dtype=dt)
    dA = bl.bl_ste_grad_input(dY.torch(DEV), to_dev(oracle.pack_ternary(codes)),
                              to_dev(np.array([g], np.float32))).cpu().numpy()
    ref = oracle.ste_grad_input(dY.f32, codes, g)
    S = float(g) * (np.abs(dY.f32.astype(np.float64)) @ np.abs(codes.astype(np.float64)))
    assert np.all(np.abs(dA - ref) <= 2.0 ** -7 * S + 1e-30), np.max(np.abs(dA - ref) - 2.0 ** -7 * S)


@pytest.mark.parametrize("M,N,K,dt", CASES)
def test_ste_grad_weight(bl, M, N, K, dt):
    W, codes, g, Aq, gA, dY = _problem(M, N, K, seed=3 * M + N, dy_dtype=dt)
    Wd = W.torch(DEV)
    dW = bl.bl_ste_grad_weight(dY.torch(DEV), to_dev(Aq), to_dev(gA), Wd,
                               to_dev(np.array([g], np.float32)), EPS).cpu().numpy()
    ref = oracle.ste_grad_weight(dY.f32, Aq, gA, W.f32, g, EPS)
    mask = oracle.ste_weight_mask(W.f32, g, EPS)
    assert np.all(dW[mask == 0] == 0.0)
    A_hat = gA.astype(np.float64)[:, None] / 127.0 * Aq
    S = mask * (np.abs(dY.f32.astype(np.float64)).T @ np.abs(A_hat))
    assert np.all(np.abs(dW - ref) <= 2.0 ** -7 * S + 1e-30), np.max(np.abs(dW - ref) - 2.0 ** -7 * S)
    assert 0.0 < mask.mean() < 1.0


def test_ste_mask_boundary(bl):
    """Latent weights at ±(γ+ε) keep their gradient, one ulp beyond drops it."""
    M, N, K = 8, 64, 64
    W, codes, g, Aq, gA, dY = _problem(M, N, K, seed=5, dy_dtype="f32")
    Wf = W.f32.copy()
    gg = np.float32(np.float32(g) + np.float32(EPS))
    Wf[0, :4] = [gg, -gg, np.nextafter(gg, np.float32(np.inf)), -np.nextafter(gg, np.float32(np.inf))]
    # keep γ as passed (the mask uses the γ given, whatever W's mean is now)
    dW = bl.bl_ste_grad_weight(to_dev(dY.f32), to_dev(Aq), to_dev(gA), to_dev(Wf),
                               to_dev(np.array([g], np.float32)), EPS).cpu().numpy()
    ref = oracle.ste_grad_weight(dY.f32, Aq, gA, Wf, g, EPS)
    assert np.all(dW[0, 2:4] == 0.0) and np.all(ref[0, 2:4] == 0.0)
    assert np.all(dW[0, :2] != 0.0) and np.all(ref[0, :2] != 0.0)


def test_ste_full_size_sampled(bl):
    """The benchmark's shape, 2048 tokens × 4096 × 4096 (two CTAs per SM, 256
    output tiles), in the launch form bench.py times. Every output row is
    independent of the others, so the oracle computes three sampled rows of
    each gradient from the same inputs: dA rows from the matching dY rows,
    dW rows from the matching dY columns and latent weight rows."""
    M, N, K = 2048, 4096, 4096
    W, codes, g, Aq, gA, dY = _problem(M, N, K, seed=11, dy_dtype="bf16")
    gd = to_dev(np.array([g], np.float32))
    dA = bl.bl_ste_grad_input(dY.torch(DEV), to_dev(oracle.pack_ternary(codes)), gd).cpu().numpy()
    dW = bl.bl_ste_grad_weight(dY.torch(DEV), to_dev(Aq), to_dev(gA), W.torch(DEV), gd,
                               EPS).cpu().numpy()
    rows_m = [0, 777, M - 1]
    ref_a = oracle.ste_grad_input(np.ascontiguousarray(dY.f32[rows_m]), codes, g)
    S_a = float(g) * (np.abs(dY.f32[rows_m].astype(np.float64)) @ np.abs(codes.astype(np.float64)))
    assert np.all(np.abs(dA[rows_m] - ref_a) <= 2.0 ** -7 * S_a + 1e-30)
    rows_n = [0, 1500, N - 1]
    dY_n = np.ascontiguousarray(dY.f32[:, rows_n])
    W_n = np.ascontiguousarray(W.f32[rows_n])
    ref_w = oracle.ste_grad_weight(dY_n, Aq, gA, W_n, g, EPS)
    mask = oracle.ste_weight_mask(W_n, g, EPS)
    assert np.all(dW[rows_n][mask == 0] == 0.0)
    A_hat = gA.astype(np.float64)[:, None] / 127.0 * Aq
    S_w = mask * (np.abs(dY_n.astype(np.float64)).T @ np.abs(A_hat))
    assert np.all(np.abs(dW[rows_n] - ref_w) <= 2.0 ** -7 * S_w + 1e-30)
