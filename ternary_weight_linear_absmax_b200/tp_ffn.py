"""Tensor-parallel ternary FFN block over ranks (torch.distributed).

The hidden dimension H of the block (BitLinear up K → H, ReLU², per-token
requantisation, BitLinear down H → K) is split into contiguous shards of a
multiple of 64: the up-projection is column-parallel, the down-projection
row-parallel. Per forward, one all-reduce(MAX) of M fp32 values makes γ_r
(the maximum is exact, so it equals the unsharded γ_r bit for bit) and one
all-reduce(SUM) of the INT32 partial down-projections [M, K] makes the
exact accumulators (integer addition does not depend on order), so the
sharded block returns exactly what bl_ffn_relu2 returns on one GPU.

Every arithmetic step runs in the CUDA library (bl_ffn_tp_up,
bl_ffn_tp_down, bl_dequant_i32); this module only shards the packed
weights and sequences the collectives (NCCL over NVLink on GPUs). The
``ops`` and ``all_reduce`` hooks exist so that the host-side logic can be
exercised with any compute backend and process group (the CPU tests use
gloo).

The pages describe no multi-GPU scheme; this is the plainest composition
of their single-GPU formulas over a split H.
"""
from __future__ import annotations

from dataclasses import dataclass


def shard_range(H: int, world: int, rank: int) -> tuple[int, int]:
    """[h0, h1) of rank `rank`: H split into `world` shards of whole 64-wide
    units, sizes differing by at most one unit, in rank order."""
    if H % 64 != 0 or H <= 0:
        raise ValueError("H must be a positive multiple of 64")
    units = H // 64
    if world > units:
        raise ValueError(f"cannot split {units} units of 64 over {world} ranks")
    base, rem = divmod(units, world)
    start = rank * base + min(rank, rem)
    size = base + (1 if rank < rem else 0)
    return 64 * start, 64 * (start + size)


def shard_packed(W_up_packed, W_down_packed, H: int, world: int, rank: int):
    """This rank's contiguous copies of the packed weights: rows [h0, h1) of
    W_up [H, K/4] and byte columns [h0/4, h1/4) of W_down [K, H/4] (h0 is a
    multiple of 64, so no 32-bit word of 16 codes is split)."""
    h0, h1 = shard_range(H, world, rank)
    return W_up_packed[h0:h1].contiguous(), W_down_packed[:, h0 // 4:h1 // 4].contiguous()


def _cuda_ops():
    import ternary_weight_linear_absmax_b200 as bl
    return bl.bl_ffn_tp_up, bl.bl_ffn_tp_down, bl.bl_dequant_i32


def _dist_all_reduce(group):
    import torch.distributed as dist

    def reduce(t, op: str):
        dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM,
                        group=group)
        return t
    return reduce


@dataclass
class TensorParallelFFN:
    """One rank's part of the block: its weight shards and the two scales."""
    W_up_r: object
    gamma_up: object
    W_down_r: object
    gamma_down: object
    eps: float = 1e-5
    group: object = None
    ops: tuple | None = None        # (up, down, dequant); default: the CUDA library
    all_reduce: object = None       # (tensor, "max" | "sum") -> tensor; default: torch.distributed

    def forward(self, X, out_dtype=None):
        up, down, dequant = self.ops if self.ops is not None else _cuda_ops()
        reduce = self.all_reduce if self.all_reduce is not None else _dist_all_reduce(self.group)
        acc_up, gamma_x, rmax = up(X, self.W_up_r, self.gamma_up, self.eps)
        gamma_r = reduce(rmax, "max")
        acc_down = down(acc_up, gamma_x, self.gamma_up, gamma_r, self.W_down_r, self.eps)
        acc_down = reduce(acc_down, "sum")
        if out_dtype is None:
            return dequant(acc_down, gamma_r, self.gamma_down)
        return dequant(acc_down, gamma_r, self.gamma_down, out_dtype=out_dtype)
