"""Host-side logic of the tensor-parallel FFN block (tp_ffn.py) on CPU.

Shard ranges, and a 2- and 3-rank gloo run of TensorParallelFFN.forward in
which each rank computes its shard with the CPU oracle's arithmetic (a
stand-in for the CUDA steps, which need a GPU) and the real
torch.distributed all-reduces combine them: the sharded block must give the
unsharded oracle block's INT32 down-projection and output exactly. The
arithmetic of the CUDA steps themselves is checked on the GPU.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

EPS = 1e-5
M, K, H = 3, 256, 640


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_shard_ranges():
    from ternary_weight_linear_absmax_b200.tp_ffn import shard_range
    for H_, world in ((11008, 2), (11008, 3), (11008, 8), (640, 10), (64, 1)):
        spans = [shard_range(H_, world, r) for r in range(world)]
        assert spans[0][0] == 0 and spans[-1][1] == H_
        for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
            assert a1 == b0
        sizes = [b - a for a, b in spans]
        assert all(s % 64 == 0 and s > 0 for s in sizes)
        assert max(sizes) - min(sizes) <= 64
    with pytest.raises(ValueError):
        shard_range(640, 11, 0)
    with pytest.raises(ValueError):
        shard_range(100, 2, 0)


def _problem():
    import oracle
    import synth_inputs as si
    Wu = si.weights(H, K, seed=1).f32
    Wd = si.weights(K, H, seed=2).f32
    cu, gu = oracle.quant_weights(Wu, EPS)
    cd, gd = oracle.quant_weights(Wd, EPS)
    X = si.activations(M, K, seed=3, outliers=True).f32
    return X, cu, gu, cd, gd


def _oracle_ops():
    """CPU stand-ins for bl_ffn_tp_up / bl_ffn_tp_down / bl_dequant_i32 with
    the oracle's fp32 arithmetic (torch CPU tensors in and out)."""
    import oracle

    def up(X, cu_r, gu, eps):
        Xq, gX = oracle.quant_acts(X.numpy(), eps)
        acc = oracle.zero_gemm(Xq, cu_r.numpy())
        h = oracle.dequant_f32(acc, gX, gu)
        r = np.maximum(h, np.float32(0)) * np.maximum(h, np.float32(0))
        return torch.from_numpy(acc), torch.from_numpy(gX), torch.from_numpy(r.max(axis=1))

    def down(acc_up, gX, gu, gR, cd_r, eps):
        h = oracle.dequant_f32(acc_up.numpy(), gX.numpy(), gu)
        r = (np.maximum(h, np.float32(0)) * np.maximum(h, np.float32(0))).astype(np.float32)
        s = (np.float32(127.0) / (gR.numpy() + np.float32(eps))).astype(np.float32)
        q = np.clip(np.rint((r * s[:, None]).astype(np.float32)), -128, 127).astype(np.int8)
        return torch.from_numpy(oracle.zero_gemm(q, cd_r.numpy()))

    def dequant(acc, gR, gd):
        return torch.from_numpy(oracle.dequant(acc.numpy(), gR.numpy(), gd))

    return up, down, dequant


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from ternary_weight_linear_absmax_b200.tp_ffn import TensorParallelFFN, shard_range
        oracle.build()
        X, cu, gu, cd, gd = _problem()
        h0, h1 = shard_range(H, world, rank)
        block = TensorParallelFFN(torch.from_numpy(cu[h0:h1].copy()), gu,
                                  torch.from_numpy(cd[:, h0:h1].copy()), gd, eps=EPS,
                                  ops=_oracle_ops())
        Y = block.forward(torch.from_numpy(X))
        q.put((rank, Y.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_block_equals_unsharded(world):
    import oracle
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    res = sorted((q.get(timeout=10) for _ in range(world)), key=lambda t: t[0])
    X, cu, gu, cd, gd = _problem()
    ref = oracle.ffn_relu2(X, cu, gu, cd, gd, EPS)["Y"]
    for rank, Y in res:
        np.testing.assert_array_equal(Y, ref)  # every rank holds the full, exact result
