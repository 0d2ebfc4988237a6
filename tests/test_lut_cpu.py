"""Host table-lookup contraction (libbitlinear_lut_cpu.so) against the oracle.

"BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM", section "Como o
ecossistema bitnet.cpp acelera inferência em CPUs e borda?": 81 pre-summed
entries per block of 4 activations, indexed by the 4 ternary weights. The
integer results must equal the oracle's add/subtract/skip contraction bit for
bit on every instruction-set path this CPU has; the table must follow the
figure's index order (0 = all -1, 40 = all 0, 80 = all +1).
"""
import numpy as np
import pytest

import oracle
import synth_inputs as si
from conftest import read_golden

EPS = 1e-5


@pytest.fixture(scope="module")
def lc():
    from ternary_weight_linear_absmax_b200 import build as b
    from ternary_weight_linear_absmax_b200 import lut_cpu
    b.build_cpu()
    oracle.build()
    return lut_cpu


def isas(lc):
    out = [lc.ISA_SCALAR]
    if lc.best_isa() >= lc.ISA_AVX2:
        out.append(lc.ISA_AVX2)
    if lc.best_isa() >= lc.ISA_AVX512:
        out.append(lc.ISA_AVX512)
    return out


def random_codes(N, K, seed):
    return (np.floor(si.uniform(seed, N * K).reshape(N, K) * 3.0).astype(np.int8) - 1)


def random_int8(M, K, seed):
    return (-127 + np.floor(si.uniform(seed, M * K).reshape(M, K) * 255)).astype(np.int8)


def test_table_follows_figure_index_order(lc):
    g = read_golden("lut_index_convention.txt")
    a = np.array([42, -18, 105, -7], np.int8)
    t = lc.table(a)
    assert t.size == g["entries"][0]
    assert t[g["index_all_minus"][0]] == -int(a.astype(int).sum())
    assert t[g["index_all_zero"][0]] == 0
    assert t[g["index_all_plus"][0]] == int(a.astype(int).sum())
    # every entry is the signed sum of its base-3 digits (first weight most significant)
    for idx in range(81):
        d = [idx // 27, (idx // 9) % 3, (idx // 3) % 3, idx % 3]
        assert t[idx] == sum((di - 1) * int(ai) for di, ai in zip(d, a))


def test_worked_example(lc):
    g = read_golden("zero_gemm_worked_example.txt")
    a = np.zeros((1, 16), np.int8)
    w = np.zeros((3, 16), np.int8)
    a[0, :8] = g["activations"]
    w[:, :8] = g["weights"]
    idx = lc.index_from_packed(oracle.pack_ternary(w), 16)
    for isa in isas(lc):
        acc = lc.lut_gemm(a, idx, 3, threads=1, isa=isa)
        assert np.all(acc == g["final_acc"][0])


@pytest.mark.parametrize("M,K,N", [(1, 64, 1), (1, 2560, 6912), (3, 192, 37), (5, 4096, 300),
                                   (2, 11008, 17), (4, 512, 256)])
def test_lut_gemm_bit_exact(lc, M, K, N):
    Aq = random_int8(M, K, seed=M + K)
    codes = random_codes(N, K, seed=N + 3 * K)
    idx = lc.index_from_packed(oracle.pack_ternary(codes), K)
    ref = oracle.zero_gemm(Aq, codes)
    for isa in isas(lc):
        for threads in (1, 3):
            np.testing.assert_array_equal(lc.lut_gemm(Aq, idx, N, threads=threads, isa=isa), ref)


def test_lut_gemm_extremes(lc):
    K, N = 4096, 64
    Aq = np.full((2, K), 127, np.int8)
    Aq[1] = -127
    codes = np.ones((N, K), np.int8)
    codes[N // 2:] = -1
    idx = lc.index_from_packed(oracle.pack_ternary(codes), K)
    ref = oracle.zero_gemm(Aq, codes)
    assert abs(int(ref.max())) == 127 * K
    for isa in isas(lc):
        np.testing.assert_array_equal(lc.lut_gemm(Aq, idx, N, isa=isa), ref)


def test_bitlinear_lut_matches_oracle(lc):
    """Decode workload (1 token, 2560 → 6912, 1 % ×20 outliers) and the
    single-layer workload: int8 tokens and γ_A equal, fp32 output close."""
    for M, K, N, outl in ((1, 2560, 6912, True), (4, 512, 256, False)):
        W = si.weights(N, K, seed=0, dtype="bf16")
        codes, g = oracle.quant_weights(W.f32, EPS)
        A = si.activations(M, K, seed=0, outliers=outl, dtype="bf16")
        idx = lc.index_from_packed(oracle.pack_ternary(codes), K)
        Y, q, gA = lc.bitlinear_lut(A.f32, idx, g, N, EPS)
        ref = oracle.bitlinear(A.f32, codes, g, EPS)
        np.testing.assert_array_equal(q, ref["Aq"])
        np.testing.assert_array_equal(gA, ref["gammaA"])
        np.testing.assert_allclose(Y, ref["Y"], rtol=1e-3, atol=1e-5)


def test_invalid_code_refused(lc):
    packed = np.full((1, 16), 0xFF, np.uint8)  # every code 3
    with pytest.raises(ValueError):
        lc.index_from_packed(packed, 64)


def test_header_symbols_exported(lc):
    """Every function include/bitlinear_lut_cpu.h declares is exported."""
    import os
    import re
    from conftest import ROOT
    text = open(os.path.join(ROOT, "include", "bitlinear_lut_cpu.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    syms = sorted(set(re.findall(r"\b(blc_[a-z0-9_]+)\s*\(", text)))
    assert len(syms) == 6
    L = lc.load()
    for s in syms:
        assert hasattr(L, s), s
