"""Lookup-table decode GEMV (bl_pack_lut_index, bl_linear_lut) through the C
ABI, against the oracle.

"BitNet b1.58 — quantização ternária, BitLinear, Zero-GEMM", figure "Fluxo de
Execução com Lookup Table (LUT-GEMM)": 81 pre-summed entries per block of 4
activations, index 27·d0 + 9·d1 + 3·d2 + d3 (d = w + 1, index 0 = all -1,
40 = all 0, 80 = all +1). The index bytes must follow that order exactly,
the INT32 result must equal the oracle's contraction of the oracle's int8
token, and the dequantised output must equal bl_linear's bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from conftest import read_golden
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


def test_index_bytes_follow_figure(bl):
    g = read_golden("lut_index_convention.txt")
    N, K = 300, 256
    codes = (np.floor(si.uniform(5, N * K).reshape(N, K) * 3.0).astype(np.int8) - 1)
    codes[0, :4], codes[0, 4:8], codes[0, 8:12] = -1, 0, 1
    idx = bl.bl_pack_lut_index(to_dev(oracle.pack_ternary(codes))).cpu().numpy()
    d = (codes.astype(np.int32) + 1).reshape(N, K // 4, 4)
    expect = 27 * d[..., 0] + 9 * d[..., 1] + 3 * d[..., 2] + d[..., 3]
    np.testing.assert_array_equal(idx, expect)
    assert idx[0, 0] == g["index_all_minus"][0]
    assert idx[0, 1] == g["index_all_zero"][0]
    assert idx[0, 2] == g["index_all_plus"][0]


@pytest.mark.parametrize("K,N,dt", [(2560, 6912, "bf16"), (4096, 1000, "f32"), (64, 33, "bf16"),
                                    (8192, 4096, "bf16")])
def test_linear_lut(bl, K, N, dt):
    W = si.weights(N, K, seed=K % 97, dtype="bf16")
    codes, g = oracle.quant_weights(W.f32, EPS)
    packed = to_dev(oracle.pack_ternary(codes))
    widx = bl.bl_pack_lut_index(packed)
    gamma = to_dev(np.array([g], np.float32))
    A = si.activations(1, K, seed=K % 89, outliers=True, dtype=dt)
    acc = bl.bl_linear_lut(A.torch(DEV), widx, gamma, EPS, raw=True).cpu().numpy()
    Aq, gA = oracle.quant_acts(A.f32, EPS)
    np.testing.assert_array_equal(acc, oracle.zero_gemm(Aq, codes))
    for out in (torch.float32, torch.bfloat16):
        Yl = bl.bl_linear_lut(A.torch(DEV), widx, gamma, EPS, out_dtype=out)
        Y2 = bl.bl_linear(A.torch(DEV), packed, gamma, EPS, out_dtype=out)
        assert torch.equal(Yl, Y2)
        assert_close(Yl.float().cpu().numpy(), oracle.bitlinear(A.f32, codes, g, EPS)["Y"],
                     out == torch.float32)


def test_linear_lut_refuses_tables_beyond_shared_memory(bl):
    """K = 11008 needs 2752 · 41 int16 table entries (220 KB) per token: more
    than a CTA's shared memory next to its weights, so the call is refused."""
    K, N = 11008, 256
    widx = torch.zeros((N, K // 4), dtype=torch.uint8, device=DEV)
    A = torch.zeros((1, K), dtype=torch.bfloat16, device=DEV)
    g = torch.ones((1,), dtype=torch.float32, device=DEV)
    with pytest.raises(bl.BitLinearError) as e:
        bl.bl_linear_lut(A, widx, g, EPS)
    assert e.value.status == 2
