"""bl_linear_noalloc: the BitLinear entry point for callers that cannot
allocate device memory (for example a plugin whose host runtime owns all
device memory and passes in only inputs and outputs, or a serving loop that
must not call cudaMalloc on its hot path). Its scratch is a fixed 4 MiB array
inside the library instead of a caller-provided workspace.

Checked through the C ABI against the ordinary bl_linear on two calls in a
row (the second call reuses the array the first one left behind), within the
bf16 tolerance of the parity tests, and against the CPU oracle as well; sizes
whose scratch would not fit must be refused before anything runs. This file
is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth_inputs as si

pytestmark = pytest.mark.gpu

EPS = 1e-5
BL_OK, BL_ERR_WORKSPACE, BL_BF16 = 0, 8, 1


@pytest.fixture(scope="module")
def lib():
    from ternary_weight_linear_absmax_b200 import _lib
    return _lib.load()


def _packed(K, N, seed):
    import ternary_weight_linear_absmax_b200 as bl
    W = si.weights(N, K, seed=seed, dtype="bf16").torch("cuda")
    return bl.bl_quant_weights(W, EPS)


def _oracle_codes(K, N, seed):
    import oracle
    return oracle.quant_weights(si.weights(N, K, seed=seed, dtype="bf16").f32, EPS)


def _reference(lib, A, packed, gamma, relu2):
    """Output of the existing entry point, bl_linear, with a torch workspace."""
    M, K = A.shape
    N = packed.shape[0]
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    nws = lib.bl_linear_workspace_bytes(M, K, N)
    ws = torch.empty(max(nws, 1), dtype=torch.uint8, device="cuda")
    st = lib.bl_linear(A.data_ptr(), BL_BF16, M, K, packed.data_ptr(), gamma.data_ptr(), N,
                       EPS, int(relu2), Y.data_ptr(), BL_BF16, ws.data_ptr() if nws else None,
                       nws, torch.cuda.current_stream().cuda_stream)
    assert st == BL_OK
    return Y


def _noalloc(lib, A, packed, gamma, relu2, Y):
    M, K = A.shape
    N = packed.shape[0]
    return lib.bl_linear_noalloc(A.data_ptr(), BL_BF16, M, K, packed.data_ptr(), gamma.data_ptr(),
                                 N, EPS, int(relu2), Y.data_ptr(), BL_BF16,
                                 torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("M,K,N", [(64, 512, 384), (300, 2560, 640), (3, 4096, 512)])
def test_noalloc_matches_bl_linear_two_calls(lib, M, K, N):
    import oracle
    packed, gamma = _packed(K, N, seed=M)
    codes, g = _oracle_codes(K, N, seed=M)
    for call, relu2 in enumerate((False, True)):  # two calls in a row
        Ah = si.activations(M, K, seed=10 * M + call, dtype="bf16")
        A = Ah.torch("cuda")
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(lib, A, packed, gamma, relu2, Y) == BL_OK
        ref = _reference(lib, A, packed, gamma, relu2)
        torch.cuda.synchronize()
        got = Y.float().cpu().numpy()
        np.testing.assert_allclose(got, ref.float().cpu().numpy(), rtol=1e-2, atol=0.0)
        # and against the independent CPU oracle on the same inputs
        np.testing.assert_allclose(got, oracle.bitlinear(Ah.f32, codes, g, EPS, relu2=relu2)["Y"],
                                   rtol=1e-2, atol=0.0)
    assert lib.bl_check_device_error(torch.cuda.current_stream().cuda_stream) == BL_OK


def test_noalloc_refuses_scratch_beyond_4mib(lib):
    M, K, N = 2048, 4096, 256  # needs 8 MiB of quantised tokens
    assert lib.bl_linear_workspace_bytes(M, K, N) > (4 << 20)
    packed, gamma = _packed(K, N, seed=1)
    A = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    Y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(lib, A, packed, gamma, False, Y) == BL_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((Y == 7.0).all())  # nothing ran
    assert "workspace" in lib.bl_status_string(BL_ERR_WORKSPACE).decode()


def test_noalloc_long_rows():
    """Three tokens of 25,600 inputs: too long a row for the fused GEMV, so
    the call takes the quantiser and the warp-level kernel on its fixed
    scratch, against the oracle."""
    import oracle
    import ternary_weight_linear_absmax_b200 as bl
    from parity_helpers import assert_close
    M, K, N = 3, 25600, 256
    codes, g = _oracle_codes(K, N, seed=71)
    A = si.activations(M, K, seed=72, outliers=True, dtype="bf16")
    Y = bl.bl_linear_noalloc(A.torch("cuda"), torch.from_numpy(oracle.pack_ternary(codes)).cuda(),
                             torch.tensor([g], dtype=torch.float32, device="cuda"), EPS)
    assert_close(Y.float().cpu().numpy(), oracle.bitlinear(A.f32, codes, g, EPS)["Y"], False)
