"""Seeded synthetic inputs for the BitLinear tests and benchmark.

This module holds none of the method's arithmetic: it only draws numbers.
Both the CPU oracle and the CUDA path are fed from it, so neither side
generates its own inputs.

Recipe (published methods, own code):
  * splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014) as a counter-based stream: output i of stream
    ``seed`` is mix(seed + (i + 1) * 0x9E3779B97F4A7C15).
  * uniform double u = ((z >> 11) + 0.5) * 2**-53, in (0, 1).
  * Box–Muller (1958): pair p uses (u[2p], u[2p+1]); normal 2p is
    r*cos(2*pi*u2), normal 2p+1 is r*sin(2*pi*u2), r = sqrt(-2 ln u1).
  * values are scaled in double, rounded to fp32 (round-to-nearest-even),
    then, for bf16 tensors, fp32 is rounded to bf16 (round-to-nearest-even).
  * outlier channels: round(0.01*K) columns chosen by a Fisher–Yates shuffle
    driven by stream seed+2; those columns are multiplied by 20 (in double,
    before rounding) for every token.
  * streams: weights use ``seed``, activations ``seed + 1``, outlier
    selection ``seed + 2``.
"""
from __future__ import annotations

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def splitmix64(seed: int, start: int, count: int) -> np.ndarray:
    """Outputs start .. start+count-1 of the splitmix64 stream ``seed``."""
    with np.errstate(over="ignore"):
        idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + idx * GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform(seed: int, count: int, start: int = 0) -> np.ndarray:
    z = splitmix64(seed, start, count)
    return ((z >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normal(seed: int, count: int, chunk: int = 1 << 22) -> np.ndarray:
    """``count`` standard normals (float64) of stream ``seed``."""
    out = np.empty(count, np.float64)
    npairs = (count + 1) // 2
    p0 = 0
    while p0 < npairs:
        p1 = min(npairs, p0 + chunk)
        u = uniform(seed, 2 * (p1 - p0), start=2 * p0)
        u1, u2 = u[0::2], u[1::2]
        r = np.sqrt(-2.0 * np.log(u1))
        t = 2.0 * np.pi * u2
        z = np.empty(2 * (p1 - p0), np.float64)
        z[0::2] = r * np.cos(t)
        z[1::2] = r * np.sin(t)
        n0, n1 = 2 * p0, min(count, 2 * p1)
        out[n0:n1] = z[: n1 - n0]
        p0 = p1
    return out


def fisher_yates(seed: int, n: int) -> np.ndarray:
    """Permutation of range(n): for i = n-1 .. 1 swap i with j = floor(u*(i+1))."""
    perm = np.arange(n, dtype=np.int64)
    u = uniform(seed, max(n - 1, 0))
    for t, i in enumerate(range(n - 1, 0, -1)):
        j = int(u[t] * (i + 1))
        perm[i], perm[j] = perm[j], perm[i]
    return perm


def outlier_channels(seed: int, K: int, frac: float = 0.01) -> np.ndarray:
    n_out = int(round(frac * K))
    return np.sort(fisher_yates(seed + 2, K)[:n_out])


# ---------------------------------------------------------------------------
# fp32 <-> bf16 bit conversions (storage formats only).

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round-to-nearest-even (no NaNs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp32, exact."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


class Tensor:
    """A host tensor as generated: fp32 values plus, for bf16, the bit patterns.
    ``f32`` is always the exact value the kernels see (bf16 widened)."""

    def __init__(self, f32: np.ndarray, dtype: str, bits: np.ndarray | None = None):
        self.f32 = f32
        self.dtype = dtype
        self.bits = bits

    @property
    def shape(self):
        return self.f32.shape

    def torch(self, device="cpu"):
        import torch
        if self.dtype == "bf16":
            t = torch.from_numpy(self.bits.view(np.int16).copy()).view(torch.bfloat16)
        else:
            t = torch.from_numpy(self.f32.copy())
        return t.to(device)


def _finish(vals: np.ndarray, dtype: str) -> Tensor:
    f = vals.astype(np.float32)
    if dtype == "f32":
        return Tensor(f, "f32")
    if dtype == "bf16":
        bits = f32_to_bf16_bits(f)
        return Tensor(bf16_bits_to_f32(bits), "bf16", bits)
    raise ValueError(dtype)


def weights(N: int, K: int, seed: int = 0, sigma: float = 0.02, dtype: str = "f32") -> Tensor:
    """W [N, K] ~ N(0, sigma^2), stream ``seed``."""
    v = normal(seed, N * K).reshape(N, K) * sigma
    return _finish(v, dtype)


def activations(M: int, K: int, seed: int = 0, outliers: bool = True,
                scale: float = 20.0, dtype: str = "f32") -> Tensor:
    """A [M, K] ~ N(0, 1), stream ``seed + 1``; with ``outliers`` the
    round(0.01*K) channels picked by stream ``seed + 2`` are scaled by 20."""
    v = normal(seed + 1, M * K).reshape(M, K)
    if outliers:
        ch = outlier_channels(seed, K)
        v[:, ch] *= scale
    return _finish(v, dtype)


# The five workloads (shapes and distributions) the library is exercised on.
CONFIGS = {
    "single": dict(M=4, K=512, N=256, w_dtype="f32", a_dtype="f32", outliers=False,
                   out="f32", eps=1e-5),
    "decode": dict(M=1, K=2560, N=6912, w_dtype="bf16", a_dtype="bf16", outliers=True,
                   out="bf16", eps=1e-5),
    "small_batch": dict(M=16, K=4096, N=11008, w_dtype="bf16", a_dtype="bf16", outliers=True,
                        out="bf16", eps=1e-5),
    "prefill": dict(M=2048, K=4096, N=4096, w_dtype="bf16", a_dtype="bf16", outliers=True,
                    out="bf16", eps=1e-5),
    "ffn": dict(M=(1, 64, 512), K=4096, H=11008, w_dtype="bf16", a_dtype="bf16", outliers=True,
                out="bf16", eps=1e-5),
}
