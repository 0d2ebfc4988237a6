"""Comparison helpers shared by the GPU parity tests.

Integers the path decides (ternary codes, int8 tokens, requantised int8,
INT32 accumulators) must equal the oracle's bit for bit. The one allowance: a
quantiser element may differ where the fp32 value being rounded lies within
one ulp of a k + 1/2 boundary (the pages do not fix the rounding of such
ties beyond "Round"). Such elements are counted, must stay at most 1e-6 of
the elements compared, and every count (zero included) is recorded in
``EXEMPTIONS`` and printed in pytest's terminal summary.
"""
from __future__ import annotations

import numpy as np

import oracle

EPS = 1e-5

# (what, differing elements, elements compared), appended by every check.
EXEMPTIONS: list[tuple[str, int, int]] = []


def near_half_boundary(x: np.ndarray) -> np.ndarray:
    """|x| within one ulp of a k + 1/2 rounding boundary (fp32)."""
    x = np.abs(x.astype(np.float32))
    b = np.floor(x) + np.float32(0.5)
    return np.abs(x - b) <= np.spacing(b)


def _exempt(got: np.ndarray, ref: np.ndarray, x: np.ndarray, what: str) -> int:
    """Count differing int8 codes; each must sit on a rounding boundary of x."""
    diff = got != ref
    nd = int(diff.sum())
    EXEMPTIONS.append((what, nd, int(ref.size)))
    if nd:
        assert np.all(np.abs(got[diff].astype(np.int32) - ref[diff].astype(np.int32)) == 1), \
            f"{what}: a code differs by more than one step"
        assert np.all(near_half_boundary(x[diff])), f"{what}: mismatch away from a rounding boundary"
        assert nd <= 1e-6 * ref.size, f"{what}: {nd} boundary exemptions of {ref.size}"
    return nd


def assert_acts_match(Aq_gpu, gA_gpu, rs_gpu, A32, eps=EPS, what="act_q"):
    """AbsMax tokens, γ_A and Σ A_q of the GPU against the oracle's
    quantise_activations_8bit on the same fp32 values."""
    Aq_gpu = np.asarray(Aq_gpu)
    Aq_ref, gA_ref = oracle.quant_acts(A32, eps)
    np.testing.assert_array_equal(np.asarray(gA_gpu), gA_ref, err_msg=f"{what}: gamma")
    s = (np.float32(127.0) / (gA_ref + np.float32(eps))).astype(np.float32)
    x = (A32.astype(np.float32) * s[:, None]).astype(np.float32)
    _exempt(Aq_gpu, Aq_ref, x, what)
    if rs_gpu is not None:
        np.testing.assert_array_equal(np.asarray(rs_gpu), Aq_gpu.astype(np.int64).sum(axis=1),
                                      err_msg=f"{what}: row sums")
    return Aq_ref, gA_ref


def assert_requant_match(Rq_gpu, gR_gpu, rs_gpu, acc_ref, gX_ref, g_up, eps=EPS, what="req_q"):
    """ReLU² requantisation of the GPU against the oracle's, both decided from
    the oracle's own up-projection accumulators."""
    Rq_gpu = np.asarray(Rq_gpu)
    Rq_ref, gR_ref = oracle.relu2_requant(acc_ref, gX_ref, g_up, eps)
    np.testing.assert_array_equal(np.asarray(gR_gpu), gR_ref, err_msg=f"{what}: gamma_r")
    h = oracle.dequant_f32(acc_ref, gX_ref, g_up)
    r = (np.maximum(h, np.float32(0)) * np.maximum(h, np.float32(0))).astype(np.float32)
    s = (np.float32(127.0) / (gR_ref + np.float32(eps))).astype(np.float32)
    x = (r * s[:, None]).astype(np.float32)
    _exempt(Rq_gpu, Rq_ref, x, what)
    if rs_gpu is not None:
        np.testing.assert_array_equal(np.asarray(rs_gpu), Rq_gpu.astype(np.int64).sum(axis=1),
                                      err_msg=f"{what}: row sums")
    return Rq_ref, gR_ref


def assert_close(got, ref, out_is_f32: bool):
    """fp32 outputs within 1e-3 rel / 1e-5 abs; bf16 outputs within 1e-2 rel."""
    got = np.asarray(got, np.float64)
    if out_is_f32:
        np.testing.assert_allclose(got, ref, rtol=1e-3, atol=1e-5)
    else:
        np.testing.assert_allclose(got, ref, rtol=1e-2, atol=0.0)
