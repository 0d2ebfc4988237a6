"""Pins for the CPU oracle: each check ties it to something other than itself
(a value the pages print, a closed form, an exact special case that reduces
to a library routine, an invariant, or brute force on tiny inputs).

Page references: [BLOG] = "BitNet b1.58 — quantização ternária, BitLinear,
Zero-GEMM"; [STUDY] = "Estudos — o dia que entendi por que ternário cabe em
um bit e meio".
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest

import synth_inputs as si
from conftest import read_golden


# ---------------------------------------------------------------------------
# Contraction (Zero-GEMM)

def test_worked_example_minus_149(orc):
    """[BLOG] §Zero-GEMM worked example: INT8 x ternary = -149, step by step."""
    g = read_golden("zero_gemm_worked_example.txt")
    a = np.array([g["activations"]], np.int8)
    w = np.array([g["weights"]], np.int8)
    assert orc.zero_gemm(a, w)[0, 0] == g["final_acc"][0] == -149
    assert orc.lut_gemm(a, w)[0, 0] == -149
    # the page's running accumulator: prefix contractions reproduce each step
    for k, expect in enumerate(g["running_acc"], start=1):
        a_k = np.zeros_like(a)
        a_k[0, :k] = a[0, :k]
        assert orc.zero_gemm(a_k, w)[0, 0] == expect


def test_zero_gemm_equals_integer_matmul(orc):
    """Textbook reduction: on ternary codes the add/sub/skip contraction is the
    ordinary integer product A_q · W_qᵀ (non-square, so a transposed operand fails)."""
    rng = np.random.default_rng(1)
    M, N, K = 5, 7, 48
    Aq = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    Wq = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    ref = Aq.astype(np.int64) @ Wq.astype(np.int64).T
    np.testing.assert_array_equal(orc.zero_gemm(Aq, Wq), ref)


def test_zero_gemm_brute_force_all_ternary_rows_k8(orc):
    """All 3^8 ternary weight rows for K=8 against a numpy dot product."""
    rows = np.array(list(itertools.product([-1, 0, 1], repeat=8)), np.int8)
    rng = np.random.default_rng(2)
    Aq = rng.integers(-127, 128, size=(3, 8)).astype(np.int8)
    Aq[0] = [127] * 8
    Aq[1] = [-127] * 8
    acc = orc.zero_gemm(Aq, rows)
    np.testing.assert_array_equal(acc, Aq.astype(np.int64) @ rows.astype(np.int64).T)
    assert acc[0].max() == 8 * 127 and acc[0].min() == -8 * 127


def test_lut_contraction_agrees(orc):
    """[BLOG] §bitnet.cpp: the 81-entry table contraction gives the same INT32."""
    g = read_golden("lut_index_convention.txt")
    assert g["entries"][0] == 3 ** 4
    # index convention: base-3 digits d = w + 1, first weight most significant
    idx = lambda w: 27 * (w[0] + 1) + 9 * (w[1] + 1) + 3 * (w[2] + 1) + (w[3] + 1)
    assert idx([-1] * 4) == g["index_all_minus"][0]
    assert idx([0] * 4) == g["index_all_zero"][0]
    assert idx([1] * 4) == g["index_all_plus"][0]
    rng = np.random.default_rng(3)
    Aq = rng.integers(-127, 128, size=(6, 256)).astype(np.int8)
    Wq = rng.integers(-1, 2, size=(40, 256)).astype(np.int8)
    np.testing.assert_array_equal(orc.lut_gemm(Aq, Wq), orc.zero_gemm(Aq, Wq))


def test_int32_accumulation_does_not_wrap(orc):
    """[BLOG] §Zero-GEMM: INT32 accumulators; a worst-case row of 11008 terms
    (|acc| = 127·11008 > int16 range) is exact."""
    K = 11008
    Aq = np.full((1, K), 127, np.int8)
    Wq = np.ones((2, K), np.int8)
    Wq[1] = -1
    acc = orc.zero_gemm(Aq, Wq)
    assert acc[0, 0] == 127 * K and acc[0, 1] == -127 * K


# ---------------------------------------------------------------------------
# Weight quantisation (AbsMean)

def test_gamma_is_per_tensor_mean(orc):
    """[BLOG] γ = (1/(n·m)) Σ|W_ij| over the whole matrix: rows of scale 1 and
    3 give γ = 2, so row 0 codes to 0 and row 1 to ±1 (per-row γ would give ±1 everywhere)."""
    W = np.array([[1.0] * 16, [-3.0] * 16], np.float32)
    codes, gamma = orc.quant_weights(W, 1e-5)
    assert gamma == np.float32(2.0)
    np.testing.assert_array_equal(codes[0], 0)
    np.testing.assert_array_equal(codes[1], -1)


def test_scaled_ternary_reproduces_itself(orc):
    """W = c·T with T ternary: W/(γ+ε) = ±1/(f+ε/c) clips to ±1, zeros stay 0."""
    rng = np.random.default_rng(4)
    T = rng.integers(-1, 2, size=(64, 96)).astype(np.int8)
    for c in (0.013, 0.5, 7.0):
        W = (c * T).astype(np.float32)
        codes, gamma = orc.quant_weights(W, 1e-5)
        np.testing.assert_array_equal(codes, T)
        f = np.count_nonzero(T) / T.size
        assert abs(float(gamma) - c * f) <= 1e-6 * c


def test_weight_rounding_threshold_exact(orc):
    """Code decision against the exact characterisation of fp32 division and
    round-half-even: Round(Clip(fl(W/g))) = sign(W) iff |W| > g·(1/2 + 2^-25)
    (quotients in (1/2, 1/2+2^-25] round to 1/2, whose tie goes to 0).
    Checked with exact rationals on values a few ulps around the boundary."""
    eps = np.float32(1e-5)
    gamma = np.float32(0.0173)
    g = np.float32(gamma + eps)
    half = np.float32(g) * np.float32(0.5)  # exact (power-of-two scale)
    vals = []
    for base in (half, -half):
        x = np.float32(base)
        for _ in range(6):
            x = np.nextafter(x, np.float32(np.inf) if base > 0 else np.float32(-np.inf))
        for _ in range(12):
            vals.append(x)
            x = np.nextafter(x, np.float32(0))
    W = np.array([vals], np.float32)
    codes = orc.ternary_codes(W, gamma, eps)[0]
    thr = Fraction(float(g)) * (Fraction(1, 2) + Fraction(1, 2 ** 25))
    expect = [0 if abs(Fraction(float(v))) <= thr else (1 if v > 0 else -1) for v in vals]
    np.testing.assert_array_equal(codes, expect)
    assert 0 in expect and 1 in expect and -1 in expect


def test_eps_in_weight_denominator(orc):
    """ε sits in the denominator: with ε = 1 and γ = 1, W/(γ+ε) = 1/2 ties to 0
    (dropping ε would give 1)."""
    W = np.ones((1, 16), np.float32)
    codes, gamma = orc.quant_weights(W, 1.0)
    assert gamma == 1.0
    np.testing.assert_array_equal(codes, 0)


def test_gaussian_weight_statistics(orc):
    """W ~ N(0, σ²): γ → σ·sqrt(2/π) and P(code = 0) → 2Φ(½·(γ+ε)/σ) − 1
    (≈ 0.310), each within 4 standard errors at 512×512."""
    N = K = 512
    sigma = 0.02
    W = si.weights(N, K, seed=0, sigma=sigma).f32
    codes, gamma = orc.quant_weights(W, 1e-5)
    n = N * K
    g_exp = sigma * math.sqrt(2 / math.pi)
    g_se = sigma * math.sqrt(1 - 2 / math.pi) / math.sqrt(n)
    assert abs(float(gamma) - g_exp) < 4 * g_se
    t = 0.5 * (float(gamma) + 1e-5) / sigma
    p0 = math.erf(t / math.sqrt(2))
    se = math.sqrt(p0 * (1 - p0) / n)
    frac0 = np.count_nonzero(codes == 0) / n
    assert abs(frac0 - p0) < 4 * se
    fp, fm = np.count_nonzero(codes == 1) / n, np.count_nonzero(codes == -1) / n
    assert abs(fp - fm) < 8 * math.sqrt(0.35 / n)
    assert set(np.unique(codes)) <= {-1, 0, 1}


def test_zero_matrix(orc):
    """γ = 0: W/ε = 0 → all codes 0, no NaN."""
    codes, gamma = orc.quant_weights(np.zeros((4, 32), np.float32), 1e-5)
    assert gamma == 0.0
    np.testing.assert_array_equal(codes, 0)


# ---------------------------------------------------------------------------
# 2-bit packing

def test_pack_layout_hand_example(orc):
    """Layout: code c = w+1; weight 16g+4j+i at bits 8i+2j of little-endian
    word g. All +1 (code 2 = 0b10 → every byte 0xAA) except k = 5
    (j=1, i=1 → bits 10..11 cleared) gives word 0xAAAAA2AA."""
    w = np.ones((1, 16), np.int8)
    w[0, 5] = -1
    p = orc.pack_ternary(w)
    assert p.shape == (1, 4)
    assert int.from_bytes(bytes(p[0]), "little") == 0xAAAAA2AA
    w2 = np.zeros((1, 16), np.int8)
    w2[0, 15] = 1  # j=3, i=3 -> bits 30..31 = code 2; others code 1 = 0b01
    assert int.from_bytes(bytes(orc.pack_ternary(w2)[0]), "little") == 0x95555555


def test_pack_roundtrip_and_size(orc):
    """Round trip; 0.25 byte per weight, i.e. the 87.5% cut against FP16 and
    the model-size column of [BLOG] §Memory Wall."""
    rng = np.random.default_rng(5)
    N, K = 37, 320
    Wq = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    p = orc.pack_ternary(Wq)
    assert p.nbytes == N * K // 4
    back, bad = orc.unpack_ternary(p, K)
    assert bad == 0
    np.testing.assert_array_equal(back, Wq)
    assert not np.any((p & 0x03) == 0x03)  # code 3 never written
    g = read_golden("memory_wall_tables.txt")
    bpw = p.nbytes / Wq.size
    assert bpw == g["bytes_per_weight_2bit"][0]
    assert 1 - bpw / 2.0 == g["traffic_reduction_vs_fp16"][0]
    assert 2.0 / (2.0 * 1.0) == g["intensity_fp16_op_per_byte"][0]
    assert 2.0 / bpw == g["intensity_2bit_op_per_byte"][0]
    for params_b, fp16_gb, int4_gb, pack_gb in g["table"]:
        assert abs(params_b * 2.0 - fp16_gb) < 1e-9
        assert abs(params_b * 0.5 - int4_gb) < 1e-9
        assert abs(params_b * bpw - pack_gb) < 1e-9


def test_unpack_flags_invalid_code(orc):
    p = np.full((1, 4), 0xFF, np.uint8)
    _, bad = orc.unpack_ternary(p, 16)
    assert bad == 16


def test_information_content_doc_pin():
    """Documentation pin: log2(3) bits of information per ternary weight; the
    2-bit code uses 3 of its 4 states; radix-3 figures as printed."""
    g = read_golden("information_content.txt")
    assert round(math.log2(3), 5) == g["log2_3_blog"][0]
    assert round(math.log2(3), 3) == g["log2_3_study"][0]
    assert 3 ** g["radix3_trits_per_byte"][0] == g["radix3_states"][0] <= 256
    assert round(8 / 5, 2) == g["radix3_bits_per_weight"][0]
    assert round(243 / 256, 3) == g["radix3_state_fraction"][0]


# ---------------------------------------------------------------------------
# Activation quantisation (AbsMax, per token)

def test_integer_activations_roundtrip(orc):
    """Integer rows in [-127,127] with row max 127: s = 127/(127+ε) and
    A·s rounds back to A."""
    rng = np.random.default_rng(6)
    A = rng.integers(-127, 128, size=(5, 64)).astype(np.float32)
    A[:, 0] = 127
    q, g = orc.quant_acts(A, 1e-5)
    np.testing.assert_array_equal(q, A.astype(np.int8))
    np.testing.assert_array_equal(g, 127.0)


def test_activation_round_half_even(orc):
    """With γ_A = 126 and ε = 1, s = 127/127 = 1 exactly, so Round sees the
    values themselves: ties go to even."""
    A = np.array([[126.0, 2.5, 3.5, -2.5, 0.5, 1.5, -0.5, -3.5, 125.5] + [0.0] * 7], np.float32)
    q, g = orc.quant_acts(A, 1.0)
    assert g[0] == 126.0
    np.testing.assert_array_equal(q[0, :9], [126, 2, 4, -2, 0, 2, 0, -4, 126])


def test_activation_scale_is_per_token(orc):
    """[BLOG] AbsMax 'dinamicamente por token': each row has its own γ_A and
    reaches ±127 at its own maximum (γ_A ≥ 253ε)."""
    A = si.activations(8, 256, seed=0, outliers=True).f32
    A[3] *= 1e-3
    q, g = orc.quant_acts(A, 1e-5)
    np.testing.assert_array_equal(g, np.abs(A).max(axis=1))
    np.testing.assert_array_equal(np.abs(q.astype(np.int32)).max(axis=1), 127)
    assert q.min() >= -127 and q.max() <= 127


def test_zero_token(orc):
    q, g = orc.quant_acts(np.zeros((2, 32), np.float32), 1e-5)
    assert np.all(q == 0) and np.all(g == 0)


# ---------------------------------------------------------------------------
# Dequantisation and the whole layer

def test_dequant_scale(orc):
    """(γ_A·γ)/127 with γ_A = 127, γ = 1 is exactly 1: y = acc."""
    acc = np.array([[-149, 0, 5, 2 ** 20]], np.int32)
    Y = orc.dequant(acc, np.array([127.0], np.float32), 1.0)
    np.testing.assert_array_equal(Y, acc.astype(np.float64))
    Y2 = orc.dequant(acc, np.array([127.0], np.float32), 1.0, relu2=True)
    np.testing.assert_array_equal(Y2, [[0.0, 0.0, 25.0, 2.0 ** 40]])


@pytest.mark.parametrize("relu2", [False, True])
def test_bitlinear_exact_special_case_equals_matmul(orc, relu2):
    """Integer activations with row max 127 and weights ±c (no zeros) are
    represented exactly by the quantisers (A_q = A, γ_A = 127, W_q = W/c,
    γ = c), so BitLinear equals the float product A·Wᵀ (numpy, float64)."""
    rng = np.random.default_rng(7)
    M, N, K = 6, 24, 160
    A = rng.integers(-127, 128, size=(M, K)).astype(np.float32)
    A[:, 7] = -127
    c = np.float32(0.03125)
    S = rng.choice(np.array([-1, 1], np.int8), size=(N, K))
    W = (c * S).astype(np.float32)
    codes, gamma = orc.quant_weights(W, 1e-5)
    assert gamma == c
    out = orc.bitlinear(A, codes, gamma, 1e-5, relu2=relu2)
    ref = A.astype(np.float64) @ W.astype(np.float64).T
    if relu2:
        ref = np.maximum(ref, 0.0) ** 2
    np.testing.assert_array_equal(out["Y"], ref)


def test_bitlinear_approximates_float_linear(orc):
    """Statistic only (the pages give no error bound): on the single-layer
    workload the quantised layer tracks A·Wᵀ; reported, loosely bounded."""
    A = si.activations(4, 512, seed=0, outliers=False).f32
    W = si.weights(256, 512, seed=0).f32
    codes, gamma = orc.quant_weights(W, 1e-5)
    Y = orc.bitlinear(A, codes, gamma, 1e-5)["Y"]
    ref = A.astype(np.float64) @ W.astype(np.float64).T
    rel = np.linalg.norm(Y - ref) / np.linalg.norm(ref)
    assert rel < 0.6


def test_dequant_matches_real_identity(orc):
    """[BLOG, Zero-GEMM section] y = Σ_k (γ·W_q)(γ_A·A_q/127). The oracle's
    fp32 path rounds three times: γ_A·γ, ÷127, acc·sc. So it must agree with
    the real value, computed from the integers in float64, to within
    3·2⁻²⁴ relative."""
    rng = np.random.default_rng(11)
    M, N = 5, 64
    acc = rng.integers(-(2 ** 20), 2 ** 20, size=(M, N)).astype(np.int32)
    gA = rng.uniform(0.1, 30.0, size=M).astype(np.float32)
    gamma = np.float32(0.0159)
    Y = orc.dequant_f32(acc, gA, gamma)
    exact = acc.astype(np.float64) * (gA.astype(np.float64)[:, None] * np.float64(gamma) / 127.0)
    rel = np.abs(Y.astype(np.float64) - exact) / np.maximum(np.abs(exact), 1e-300)
    assert rel.max() <= 3 * 2.0 ** -24
    # the float64 dequant of the oracle is the same identity up to its own roundings
    np.testing.assert_allclose(orc.dequant(acc, gA, gamma), exact, rtol=4 * 2.0 ** -53 * 8)


def test_requant_gamma_is_image_of_max_accumulator(orc):
    """ReLU² and fp32 rounding are monotone, so γ_r = max_n r equals r computed
    from the largest accumulator: γ_r = fl(fl(max(acc,0)·s)²) with
    s = fl(fl(γ_X·γ_up)/127). A row with no positive accumulator has γ_r = 0
    and codes 0."""
    rng = np.random.default_rng(12)
    M, H = 6, 320
    acc = rng.integers(-50000, 50000, size=(M, H)).astype(np.int32)
    acc[2] = -np.abs(acc[2]) - 1  # no positive value
    gX = rng.uniform(0.5, 40.0, size=M).astype(np.float32)
    g_up = np.float32(0.0173)
    q, g = orc.relu2_requant(acc, gX, g_up, 1e-5)
    for m in range(M):
        s = np.float32(np.float32(gX[m] * g_up) / np.float32(127.0))
        h = np.float32(np.float32(max(int(acc[m].max()), 0)) * s)
        assert g[m] == np.float32(h * h), m
    assert g[2] == 0 and np.all(q[2] == 0)
    assert np.all(np.abs(q.astype(np.int32)).max(axis=1)[[0, 1, 3, 4, 5]] == 127)


def test_relu2_requant_hand_case(orc):
    """ReLU² then per-token AbsMax requant, values fixed by hand:
    h = [508, 254, 0, -254] → r = [258064, 64516, 0, 0] → γ_r = 258064;
    q = [127, round(31.75·(1-δ)) = 32, 0, 0]."""
    acc = np.array([[508, 254, 0, -254]], np.int32)
    q, g = orc.relu2_requant(acc, np.array([127.0], np.float32), 1.0, 1e-5)
    assert g[0] == np.float32(258064.0)
    np.testing.assert_array_equal(q[0], [127, 32, 0, 0])


def test_ffn_exact_special_case_equals_float_ffn(orc):
    """Activations 127·e-patterns and ±1 weights keep every stage exact:
    h = X·W_upᵀ, r = relu(h)² ∈ {0, R}, requant to {0, 127}, so the block equals
    relu(X·W_upᵀ)²·W_downᵀ computed in float64."""
    rng = np.random.default_rng(8)
    M, K, H, Nout = 3, 32, 48, 16
    X = np.zeros((M, K), np.float32)
    X[:, 0] = 127
    X[:, 1] = 127
    Wup = rng.choice(np.array([-1, 1], np.int8), size=(H, K)).astype(np.float32)
    Wdn = rng.choice(np.array([-1, 1], np.int8), size=(Nout, H)).astype(np.float32)
    cu, gu = orc.quant_weights(Wup, 1e-5)
    cd, gd = orc.quant_weights(Wdn, 1e-5)
    assert gu == 1.0 and gd == 1.0
    out = orc.ffn_relu2(X, cu, gu, cd, gd, 1e-5)
    h = X.astype(np.float64) @ Wup.astype(np.float64).T
    ref = (np.maximum(h, 0) ** 2) @ Wdn.astype(np.float64).T
    np.testing.assert_array_equal(out["Y"], ref)
    assert set(np.unique(out["Rq"])) <= {0, 127}


# ---------------------------------------------------------------------------
# STE backward ([BLOG] §Zero-GEMM, Straight-Through Estimator paragraph)

def _ste_problem(orc, M=5, N=7, K=48, seed=11):
    W = si.weights(N, K, seed=seed).f32
    codes, g = orc.quant_weights(W, 1e-5)
    A = si.activations(M, K, seed=seed + 1, outliers=True).f32
    Aq, gA = orc.quant_acts(A, 1e-5)
    dY = si.activations(M, N, seed=seed + 2).f32
    return W, codes, g, A, Aq, gA, dY


def test_ste_grad_input_bilinear_identity(orc):
    """⟨dA, Â⟩ = ⟨dY, Y⟩: the activation gradient is the adjoint of the
    forward (Y from the forward oracle, Â = γ_A·A_q/127). A transposed
    operand, a dropped γ or a sign error breaks the equality."""
    W, codes, g, A, Aq, gA, dY = _ste_problem(orc)
    dA = orc.ste_grad_input(dY, codes, g)
    A_hat = gA.astype(np.float64)[:, None] / 127.0 * Aq
    Y = orc.bitlinear(A, codes, g, 1e-5)["Y"]
    lhs, rhs = float((dA * A_hat).sum()), float((dY.astype(np.float64) * Y).sum())
    assert abs(lhs - rhs) <= 1e-12 * (abs(rhs) + 1.0)


def test_ste_grad_weight_bilinear_identity(orc):
    """⟨dW, Ŵ⊙mask⟩ = ⟨dY, Y'⟩ with Y' the forward of the masked codes:
    the weight gradient is the adjoint of the forward within the clip range."""
    W, codes, g, A, Aq, gA, dY = _ste_problem(orc, seed=21)
    mask = orc.ste_weight_mask(W, g, 1e-5)
    assert 0 < mask.mean() < 1  # some weights were clipped, some not
    dW = orc.ste_grad_weight(dY, Aq, gA, W, g, 1e-5)
    assert np.all(dW[mask == 0] == 0.0)
    W_hat = float(g) * (codes * mask).astype(np.float64)
    Yp = orc.dequant(orc.zero_gemm(Aq, (codes * mask).astype(np.int8)), gA, g)
    lhs, rhs = float((dW * W_hat).sum()), float((dY.astype(np.float64) * Yp).sum())
    assert abs(lhs - rhs) <= 1e-12 * (abs(rhs) + 1.0)


def test_ste_identity_weights_pass_dY(orc):
    """W = c·I (N = K): the codes are the identity (the diagonal clips to 1,
    the rest rounds to 0) and γ = c/K, so dA = γ·dY exactly."""
    K = 64
    W = np.eye(K, dtype=np.float32) * np.float32(0.5)
    codes, g = orc.quant_weights(W, 1e-5)
    np.testing.assert_array_equal(codes, np.eye(K, dtype=np.int8))
    assert g == np.float32(0.5 / K)
    dY = si.activations(3, K, seed=4).f32
    np.testing.assert_array_equal(orc.ste_grad_input(dY, codes, g),
                                  dY.astype(np.float64) * np.float64(g))


def test_ste_mask_boundary_ulps(orc):
    """The range test is the forward's fp32 quotient: W = γ+ε gives exactly 1
    (inside), the next float above gives a quotient above 1 (outside), for
    either sign; values between are inside."""
    W = si.weights(4, 64, seed=9).f32.copy()
    g = orc.absmean_gamma(W)
    for _ in range(20):  # crafted entries barely move γ; iterate to a fixed point
        gg = np.float32(np.float32(g) + np.float32(1e-5))
        W[0, :4] = [gg, -gg, np.nextafter(gg, np.float32(np.inf)),
                    -np.nextafter(gg, np.float32(np.inf))]
        W[0, 4] = np.nextafter(gg, np.float32(0))
        g_new = orc.absmean_gamma(W)
        if g_new == g:
            break
        g = g_new
    assert np.float32(np.float32(g) + np.float32(1e-5)) == W[0, 0]
    mask = orc.ste_weight_mask(W, g, 1e-5)
    np.testing.assert_array_equal(mask[0, :5], [1, 1, 0, 0, 1])
    x = W[0, :5] / (np.float32(g) + np.float32(1e-5))
    assert x[0] == 1.0 and x[1] == -1.0 and x[2] > 1.0 and x[3] < -1.0


def test_ste_grads_match_float64_matmul(orc):
    """Special case reducing to library routines: dA = γ·(dY @ W_q) and
    dW = mask ⊙ (dYᵀ @ Â) in float64."""
    W, codes, g, A, Aq, gA, dY = _ste_problem(orc, M=9, N=13, K=64, seed=31)
    dA = orc.ste_grad_input(dY, codes, g)
    np.testing.assert_allclose(dA, float(g) * (dY.astype(np.float64) @ codes.astype(np.float64)),
                               rtol=1e-12, atol=1e-12)
    A_hat = gA.astype(np.float64)[:, None] / 127.0 * Aq
    mask = orc.ste_weight_mask(W, g, 1e-5)
    dW = orc.ste_grad_weight(dY, Aq, gA, W, g, 1e-5)
    np.testing.assert_allclose(dW, mask * (dY.astype(np.float64).T @ A_hat), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# Radix-3 storage ([BLOG] §bitnet.cpp: 5 trits per byte)

def test_radix3_all_groups_round_trip(orc):
    """Every one of the 3^5 = 243 five-weight groups packs into a distinct
    byte and unpacks to itself; 243 of 256 byte states are used (94.9 %)."""
    groups = np.array(list(itertools.product([-1, 0, 1], repeat=5)), np.int8).reshape(1, -1)
    K = groups.shape[1]  # 1215 weights = 243 groups
    packed = orc.pack_radix3(groups)
    used = packed[0, :243]
    assert len(set(used.tolist())) == 243
    back, bad = orc.unpack_radix3(packed, K)
    assert bad == 0
    np.testing.assert_array_equal(back, groups)
    g = read_golden("information_content.txt")
    assert round(len(set(used.tolist())) / 256, 3) == g["radix3_state_fraction"][0]


def test_radix3_hand_derived_bytes(orc):
    """b = Σ d_i 3^(4-i), byte = ceil(256 b / 243): all -1 → b 0 → 0;
    all 0 → b 121 → 128; all +1 → b 242 → 255; (+1,-1,-1,-1,-1) → b 162 → 171;
    (-1,-1,-1,-1,+1) → b 2 → 3 (first weight most significant)."""
    W = np.array([[-1] * 5 + [0] * 5 + [1] * 5 + [1, -1, -1, -1, -1] + [-1, -1, -1, -1, 1]], np.int8)
    packed = orc.pack_radix3(W)
    np.testing.assert_array_equal(packed[0, :5], [0, 128, 255, 171, 3])
    assert np.all(packed[0, 5:] == 128)  # padding groups: all weights 0


def test_radix3_density_and_ragged_rows(orc):
    """1.60 bits per weight when K is a multiple of 80; ragged K pads the last
    group with zeros and the row to 16 bytes; random rows round-trip."""
    g = read_golden("information_content.txt")
    assert orc.radix3_row_bytes(2560) == 512
    assert round(8 * orc.radix3_row_bytes(2560) / 2560, 2) == g["radix3_bits_per_weight"][0]
    assert orc.radix3_row_bytes(4096) == 832  # ceil(4096/5) = 820 → 832
    rng = np.random.default_rng(12)
    for K in (64, 4096, 11008, 77):
        W = rng.integers(-1, 2, size=(7, K)).astype(np.int8)
        back, bad = orc.unpack_radix3(orc.pack_radix3(W), K)
        assert bad == 0
        np.testing.assert_array_equal(back, W)
