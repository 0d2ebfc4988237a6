"""Radix-3 weight storage (5 trits per byte) and its decode GEMV through the
C ABI, against the oracle.

"BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM", section "Como o
ecossistema bitnet.cpp acelera inferência em CPUs e borda?" (3^5 = 243 ≤ 256,
1.60 bits per weight). The packed bytes must equal the oracle's packer bit
for bit; the INT32 accumulators of bl_linear_radix3 must equal the oracle's
add/subtract/skip contraction of the oracle's int8 tokens exactly, and the
dequantised output must equal bl_linear's on the 2-bit weights bit for bit
(same integers, same fp32 epilogue) and the oracle within the bf16/fp32
tolerances.
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


@pytest.mark.parametrize("N,K", [(6912, 2560), (100, 192), (4096, 4096), (11008, 4096), (37, 64)])
def test_pack_radix3_bit_exact(bl, N, K):
    codes = (np.floor(si.uniform(N + K, N * K).reshape(N, K) * 3.0).astype(np.int8) - 1)
    r3 = bl.bl_pack_radix3(to_dev(oracle.pack_ternary(codes)), K).cpu().numpy()
    np.testing.assert_array_equal(r3, oracle.pack_radix3(codes))


CASES = [(1, 2560, 6912, "bf16"), (2, 4096, 1000, "bf16"), (3, 192, 200, "f32"),
         (4, 11008, 512, "bf16"), (1, 64, 33, "f32"), (4, 2560, 6912, "bf16")]


@pytest.mark.parametrize("M,K,N,dt", CASES)
def test_linear_radix3(bl, M, K, N, dt):
    W = si.weights(N, K, seed=M + 2, dtype="bf16")
    codes, g = oracle.quant_weights(W.f32, EPS)
    packed = to_dev(oracle.pack_ternary(codes))
    r3 = bl.bl_pack_radix3(packed, K)
    gamma = to_dev(np.array([g], np.float32))
    A = si.activations(M, K, seed=M + 3, outliers=True, dtype=dt)
    acc = bl.bl_linear_radix3(A.torch(DEV), r3, gamma, EPS, raw=True).cpu().numpy()
    Aq, gA = oracle.quant_acts(A.f32, EPS)
    np.testing.assert_array_equal(acc, oracle.zero_gemm(Aq, codes))
    for out in (torch.float32, torch.bfloat16):
        Y3 = bl.bl_linear_radix3(A.torch(DEV), r3, gamma, EPS, out_dtype=out, relu2=(M == 3))
        Y2 = bl.bl_linear(A.torch(DEV), packed, gamma, EPS, out_dtype=out, relu2=(M == 3))
        assert torch.equal(Y3, Y2)
        ref = oracle.bitlinear(A.f32, codes, g, EPS, relu2=(M == 3))["Y"]
        assert_close(Y3.float().cpu().numpy(), ref, out == torch.float32)


def test_radix3_pdl_chain(bl):
    K, N = 2560, 1024
    A = si.activations(1, K, seed=0, dtype="bf16")
    At = A.torch(DEV)
    outs, refs = [], []
    mats = []
    for i in range(5):
        codes, g = oracle.quant_weights(si.weights(N, K, seed=400 + i, dtype="bf16").f32, EPS)
        mats.append((bl.bl_pack_radix3(to_dev(oracle.pack_ternary(codes)), K),
                     to_dev(np.array([g], np.float32))))
        refs.append(oracle.bitlinear(A.f32, codes, g, EPS)["Y"])
    torch.cuda.synchronize()
    for r3, gamma in mats:
        outs.append(bl.bl_linear_radix3(At, r3, gamma, EPS, pdl=True))
    torch.cuda.synchronize()
    for y, r in zip(outs, refs):
        assert_close(y.float().cpu().numpy(), r, False)
