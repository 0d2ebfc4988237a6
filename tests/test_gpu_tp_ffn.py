"""Tensor-parallel FFN steps (bl_ffn_tp_up, bl_ffn_tp_down, bl_dequant_i32)
through the C ABI on one GPU.

The g ranks are emulated in lockstep on one device: every shard's step 1,
then the MAX over the shards' rmax (what all-reduce(MAX) computes), every
shard's step 3, then the INT32 SUM of the partial down-projections (what
all-reduce(SUM) computes), then the dequantisation. No kernel waits on
another. The result must equal the unsharded bl_ffn_relu2 output bit for bit
and the oracle's INT32 down-projection exactly, for shards that take the
fused GEMV (M = 1), the warp-level MMA (M = 5, 32) and the tensor-core
(M = 64, 130) paths.
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


@pytest.fixture(scope="module")
def block():
    K, H = 1024, 2752
    cu, gu = oracle.quant_weights(si.weights(H, K, seed=1, dtype="bf16").f32, EPS)
    cd, gd = oracle.quant_weights(si.weights(K, H, seed=2, dtype="bf16").f32, EPS)
    return K, H, cu, gu, cd, gd


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("M", [1, 5, 32, 64, 130])
def test_tp_ffn_lockstep_equals_unsharded(bl, block, world, M):
    from ternary_weight_linear_absmax_b200.tp_ffn import shard_packed
    K, H, cu, gu, cd, gd = block
    pu, pd = to_dev(oracle.pack_ternary(cu)), to_dev(oracle.pack_ternary(cd))
    gu_d, gd_d = to_dev(np.array([gu], np.float32)), to_dev(np.array([gd], np.float32))
    X = si.activations(M, K, seed=70 + M, outliers=True, dtype="bf16")
    Xd = X.torch(DEV)
    shards = [shard_packed(pu, pd, H, world, r) for r in range(world)]
    ups = [bl.bl_ffn_tp_up(Xd, su, gu_d, EPS) for su, _ in shards]
    gamma_r = torch.stack([u[2] for u in ups]).amax(dim=0)           # all-reduce(MAX)
    parts = [bl.bl_ffn_tp_down(u[0], u[1], gu_d, gamma_r, sd, EPS) for u, (_, sd) in zip(ups, shards)]
    acc_down = torch.stack(parts).sum(dim=0, dtype=torch.int32)     # all-reduce(SUM)
    Y = bl.bl_dequant_i32(acc_down, gamma_r, gd_d)
    Y_full = bl.bl_ffn_relu2(Xd, pu, gu_d, pd, gd_d, EPS)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y_full), "sharded block differs from the unsharded block"
    ref = oracle.ffn_relu2(X.f32, cu, gu, cd, gd, EPS)
    np.testing.assert_array_equal(acc_down.cpu().numpy(), ref["acc_down"])
    np.testing.assert_array_equal(gamma_r.cpu().numpy(), ref["gammaR"])
    assert_close(Y.float().cpu().numpy(), ref["Y"], False)


def test_dequant_i32_fp32_and_relu2(bl):
    acc = (np.arange(-300, 300, dtype=np.int32) * 977).reshape(6, 100)
    gA = np.array([0.5, 1.0, 2.0, 3.5, 1e-3, 0.0], np.float32)
    g = np.float32(0.02)
    Y = bl.bl_dequant_i32(to_dev(acc), to_dev(gA), to_dev(np.array([g], np.float32)),
                          out_dtype=torch.float32).cpu().numpy()
    assert_close(Y, oracle.dequant(acc, gA, g), True)
    Y2 = bl.bl_dequant_i32(to_dev(acc), to_dev(gA), to_dev(np.array([g], np.float32)), relu2=True,
                           out_dtype=torch.float32).cpu().numpy()
    assert_close(Y2, oracle.dequant(acc, gA, g, relu2=True), True)


@pytest.fixture(scope="module")
def block_wide():
    K, H = 4096, 5504
    cu, gu = oracle.quant_weights(si.weights(H, K, seed=3, dtype="bf16").f32, EPS)
    cd, gd = oracle.quant_weights(si.weights(K, H, seed=4, dtype="bf16").f32, EPS)
    return K, H, cu, gu, cd, gd


@pytest.mark.parametrize("M", [64, 130])
def test_tp_ffn_wide_shards(bl, block_wide, M):
    """Wider shards (two ranks of 4096 -> 5504 -> 4096: 2752 hidden rows per
    rank, 32 K blocks in the up-projection). The block output must equal
    the unsharded block bit for bit; the oracle checks three tokens (every
    step is per token)."""
    from ternary_weight_linear_absmax_b200.tp_ffn import shard_packed
    K, H, cu, gu, cd, gd = block_wide
    pu, pd = to_dev(oracle.pack_ternary(cu)), to_dev(oracle.pack_ternary(cd))
    gu_d, gd_d = to_dev(np.array([gu], np.float32)), to_dev(np.array([gd], np.float32))
    X = si.activations(M, K, seed=90 + M, outliers=True, dtype="bf16")
    Xd = X.torch(DEV)
    shards = [shard_packed(pu, pd, H, 2, r) for r in range(2)]
    ups = [bl.bl_ffn_tp_up(Xd, su, gu_d, EPS) for su, _ in shards]
    gamma_r = torch.stack([u[2] for u in ups]).amax(dim=0)
    parts = [bl.bl_ffn_tp_down(u[0], u[1], gu_d, gamma_r, sd, EPS) for u, (_, sd) in zip(ups, shards)]
    acc_down = torch.stack(parts).sum(dim=0, dtype=torch.int32)
    Y = bl.bl_dequant_i32(acc_down, gamma_r, gd_d)
    Y_full = bl.bl_ffn_relu2(Xd, pu, gu_d, pd, gd_d, EPS)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y_full), "sharded block differs from the unsharded block"
    rows = [0, M // 2, M - 1]
    ref = oracle.ffn_relu2(X.f32[rows], cu, gu, cd, gd, EPS)
    np.testing.assert_array_equal(acc_down.cpu().numpy()[rows], ref["acc_down"])
    np.testing.assert_array_equal(gamma_r.cpu().numpy()[rows], ref["gammaR"])
    assert_close(Y.float().cpu().numpy()[rows], ref["Y"], False)
