"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.

Bar: ternary codes, int8 activations and INT32 accumulators bit-exact (a
quantiser element may differ only within one ulp of a rounding boundary; such
elements are counted and must be ≤ 1e-6 of the elements); fp32 outputs within
1e-3 relative / 1e-5 absolute, bf16 outputs within 1e-2 relative.

Workloads: the single-layer, decode, small-batch, prefill and FFN shapes,
plus small and ragged shapes that exercise tile tails. Full-size cases
compare sampled tokens × sampled output rows, which the oracle computes
one by one.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from parity_helpers import EXEMPTIONS, assert_acts_match, near_half_boundary
from parity_helpers import assert_close as _assert_close

pytestmark = pytest.mark.gpu

EPS = 1e-5
DEV = "cuda"


@pytest.fixture(scope="module")
def bl():
    import ternary_weight_linear_absmax_b200 as m
    m.load()
    return m


# ---------------------------------------------------------------------------
# helpers

def to_dev(x: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(x)).to(DEV)


def assert_codes_match(packed_gpu, W32, gamma_gpu, K):
    codes_ref, g_ref = oracle.quant_weights(W32, EPS)
    gg = np.float32(gamma_gpu)
    ulps = abs(int(gg.view(np.int32)) - int(np.float32(g_ref).view(np.int32)))
    assert ulps <= 1, f"gamma {gg} vs oracle {g_ref}"
    codes_gpu, bad = oracle.unpack_ternary(packed_gpu, K)
    assert bad == 0
    diff = codes_gpu != codes_ref
    nd = int(diff.sum())
    EXEMPTIONS.append((f"weight codes {W32.shape[0]}x{K}", nd, int(W32.size)))
    if nd:
        x = (W32[diff] / np.float32(np.float32(g_ref) + np.float32(EPS))).astype(np.float32)
        assert np.all(near_half_boundary(x)), "code mismatch away from a rounding boundary"
        assert nd <= 1e-6 * W32.size, f"{nd} boundary exemptions"
    return codes_ref, g_ref, nd


def assert_close(got, ref, out_dtype):
    _assert_close(got, ref, out_dtype == torch.float32)


def random_codes(N, K, seed):
    u = si.uniform(seed, N * K).reshape(N, K)
    return (np.floor(u * 3.0).astype(np.int8) - 1)


def random_int8(M, K, seed, lo=-127, hi=127):
    u = si.uniform(seed, M * K).reshape(M, K)
    return (lo + np.floor(u * (hi - lo + 1))).astype(np.int8)


# ---------------------------------------------------------------------------
# a1: AbsMean ternary quantisation + packing

QW_CASES = [
    (256, 512, "f32"),      # single-layer workload
    (100, 192, "bf16"),     # ragged row count, K % 128 == 64
    (6912, 2560, "bf16"),   # decode matrix
    (11008, 4096, "bf16"),  # small-batch / FFN up
    (4096, 4096, "bf16"),   # prefill
    (4096, 11008, "bf16"),  # FFN down
]


@pytest.mark.parametrize("N,K,dt", QW_CASES)
def test_quant_weights_parity(bl, N, K, dt):
    W = si.weights(N, K, seed=0, dtype=dt)
    packed, g = bl.bl_quant_weights(W.torch(DEV), EPS)
    packed = packed.cpu().numpy()
    assert packed.shape == (N, K // 4)
    codes_ref, g_ref, nd = assert_codes_match(packed, W.f32, g.item(), K)
    if np.float32(g.item()) == np.float32(g_ref):
        np.testing.assert_array_equal(packed, oracle.pack_ternary(codes_ref))


def test_quant_weights_boundary_values(bl):
    """Weights placed within a few ulps of ±(γ+ε)/2: the GPU's exact threshold
    test must reproduce the oracle's fp32 division + round-half-even."""
    N, K = 64, 256
    W = si.weights(N, K, seed=5).f32.copy()
    g = oracle.absmean_gamma(W)
    for _ in range(3):  # fixed point: crafted entries barely move γ
        half = np.float32(np.float32(g) + np.float32(EPS)) * np.float32(0.5)
        row = []
        x = half
        for _ in range(8):
            x = np.nextafter(x, np.float32(1))
        for _ in range(16):
            row.append(x)
            x = np.nextafter(x, np.float32(0))
        row = np.array(row, np.float32)
        W[0, :16], W[0, 16:32] = row, -row
        g = oracle.absmean_gamma(W)
    packed, gg = bl.bl_quant_weights(to_dev(W), EPS)
    assert np.float32(gg.item()) == np.float32(g)
    codes_ref, _ = oracle.quant_weights(W, EPS)
    np.testing.assert_array_equal(packed.cpu().numpy(), oracle.pack_ternary(codes_ref))
    assert set(np.unique(codes_ref[0, :32])) == {-1, 0, 1}


def test_quant_weights_zero_and_scaled_ternary(bl):
    Z = np.zeros((128, 128), np.float32)
    packed, g = bl.bl_quant_weights(to_dev(Z), EPS)
    assert g.item() == 0.0
    assert np.all(packed.cpu().numpy() == 0x55)  # every code 1 (w = 0)
    T = random_codes(96, 320, seed=11)
    W = (np.float32(0.37) * T).astype(np.float32)
    packed, g = bl.bl_quant_weights(to_dev(W), EPS)
    codes, bad = oracle.unpack_ternary(packed.cpu().numpy(), 320)
    np.testing.assert_array_equal(codes, T)


# ---------------------------------------------------------------------------
# a2: AbsMax per-token activation quantisation

QA_CASES = [(4, 512, "f32", False), (1, 2560, "bf16", True), (16, 4096, "bf16", True),
            (2048, 4096, "bf16", True), (7, 11008, "f32", True), (3, 64, "bf16", False)]


@pytest.mark.parametrize("M,K,dt,outl", QA_CASES)
def test_quant_acts_parity(bl, M, K, dt, outl):
    A = si.activations(M, K, seed=0, outliers=outl, dtype=dt)
    Aq, gA, rs = bl.bl_quant_acts(A.torch(DEV), EPS)
    assert_acts_match(Aq.cpu().numpy(), gA.cpu().numpy(), rs.cpu().numpy(), A.f32,
                      what=f"bl_quant_acts {M}x{K} {dt}")


def test_quant_acts_special_rows(bl):
    K = 64
    A = np.zeros((4, K), np.float32)
    A[1, :] = np.arange(-32, 32) * 3.0
    A[1, 5] = 127.0  # integer row with max 127
    A[1, 6] = -127.0
    A[2, :9] = [126.0, 2.5, 3.5, -2.5, 0.5, 1.5, -0.5, -3.5, 125.5]  # ties with eps = 1 below
    A[3, :] = 1e-30  # tiny row
    Aq, gA, rs = bl.bl_quant_acts(to_dev(A), EPS)
    assert_acts_match(Aq.cpu().numpy(), gA.cpu().numpy(), rs.cpu().numpy(), A)
    Aq1, gA1, _ = bl.bl_quant_acts(to_dev(A[2:3]), 1.0)
    np.testing.assert_array_equal(Aq1.cpu().numpy()[0, :9], [126, 2, 4, -2, 0, 2, 0, -4, 126])


# ---------------------------------------------------------------------------
# a3: INT32 contraction, bit-exact

ZG_CASES = [
    (1, 64, 128), (2, 128, 200), (3, 192, 256), (4, 512, 256),      # GEMV path
    (5, 128, 128), (16, 4096, 384), (17, 192, 200), (32, 512, 130),  # skinny path (5..32 tokens)
    (31, 1024, 256), (8, 64, 1), (24, 3200, 1500), (20, 640, 9000),
    (7, 64, 20000), (32, 4096, 4096), (32, 4096, 11008),
    # 33..64 tokens: skinny (4 m-tiles) while tiles would fill under half the SMs ...
    (33, 512, 130), (48, 3200, 1500), (64, 1024, 256),
    # ... tensor-core tiles otherwise (unsplit, and with K split in 4)
    (40, 256, 11008), (64, 4096, 4096),
    (65, 256, 200), (100, 320, 256), (128, 256, 128), (129, 640, 260),  # tensor-core path
    (256, 512, 384), (300, 384, 512), (520, 128, 136),
    (384, 128, 7680), (300, 256, 9000),  # 192-token tiles (one round instead of two of 128)
    (512, 128, 11008),  # 192-token tiles, two CTAs per SM
    (100, 192, 300), (520, 64, 136),  # K not a multiple of the 128-wide K block
]


@pytest.mark.parametrize("M,K,N", ZG_CASES)
def test_zero_gemm_exact(bl, M, K, N):
    Aq = random_int8(M, K, seed=M * 1000 + K)
    Aq[0, : min(K, 8)] = 127
    codes = random_codes(N, K, seed=N * 7 + K)
    packed = oracle.pack_ternary(codes)
    acc = bl.bl_zero_gemm(to_dev(Aq), to_dev(packed)).cpu().numpy()
    np.testing.assert_array_equal(acc, oracle.zero_gemm(Aq, codes))


def _random_shapes(count, seed):
    """Seeded shapes over every contraction path: GEMV (≤ 4 tokens), the
    warp-level kernel (5-64), tensor-core tiles of 128/192/256 tokens, one or
    two CTAs per SM, K splits, ragged N, K not a multiple of the 128-wide
    block."""
    u = si.uniform(seed, 3 * count).reshape(count, 3)
    shapes = []
    for a, b, c in u:
        M = int(1 + a ** 2 * 700)            # biased towards small M
        K = 64 * int(1 + b * 40)             # 64 .. 2560
        N = int(1 + c ** 1.5 * 12000)
        shapes.append((M, K, N))
    return shapes


@pytest.mark.parametrize("M,K,N", _random_shapes(24, seed=2024))
def test_zero_gemm_random_shapes(bl, M, K, N):
    Aq = random_int8(M, K, seed=M * 31 + K)
    codes = random_codes(N, K, seed=N * 13 + K)
    acc = bl.bl_zero_gemm(to_dev(Aq), to_dev(oracle.pack_ternary(codes))).cpu().numpy()
    np.testing.assert_array_equal(acc, oracle.zero_gemm(Aq, codes))


def _band_shapes(count, seed):
    """33..64 tokens: the tensor-core tiles take these when they (times their
    K ranges) fill at least half of the SMs, the warp-level kernel otherwise."""
    u = si.uniform(seed, 3 * count).reshape(count, 3)
    return [(int(33 + a * 31.999), 64 * int(1 + b * 50), int(1 + c * 12000)) for a, b, c in u]


@pytest.mark.parametrize("M,K,N", _band_shapes(12, seed=3364))
def test_contraction_band_33_64(bl, M, K, N):
    """Bit-exact INT32 with room for K-split partials (bl_zero_gemm), and the
    same contraction through bl_linear_q with no workspace at all (row sums
    given; γ_A = 127, γ = 1, so Y = acc exactly in fp32)."""
    Aq = random_int8(M, K, seed=M * 17 + K)
    codes = random_codes(N, K, seed=N * 29 + K)
    packed = to_dev(oracle.pack_ternary(codes))
    ref = oracle.zero_gemm(Aq, codes)
    acc = bl.bl_zero_gemm(to_dev(Aq), packed).cpu().numpy()
    np.testing.assert_array_equal(acc, ref)
    rs = to_dev(Aq.astype(np.int32).sum(axis=1).astype(np.int32))
    Y = bl.bl_linear_q(to_dev(Aq), to_dev(np.full(M, 127.0, np.float32)), packed,
                       to_dev(np.array([1.0], np.float32)), rowsum=rs,
                       out_dtype=torch.float32).cpu().numpy()
    np.testing.assert_array_equal(Y, ref.astype(np.float32))


def test_zero_gemm_extremes(bl):
    """Worst-case magnitudes: all +127 / -127 activations against all-±1 rows."""
    for M in (1, 40):
        K, N = 4096, 256
        Aq = np.full((M, K), 127, np.int8)
        Aq[M // 2:] = -127
        codes = np.ones((N, K), np.int8)
        codes[N // 2:] = -1
        codes[:, ::3] = 0
        acc = bl.bl_zero_gemm(to_dev(Aq), to_dev(oracle.pack_ternary(codes))).cpu().numpy()
        np.testing.assert_array_equal(acc, oracle.zero_gemm(Aq, codes))


def test_zero_gemm_worked_example(bl):
    """The blog's 8-element example (-149), padded to one 64-wide K block."""
    a = np.zeros((1, 64), np.int8)
    w = np.zeros((1, 64), np.int8)
    a[0, :8] = [42, -18, 105, -7, 88, 12, -64, 3]
    w[0, :8] = [1, 0, -1, 1, 0, -1, 1, -1]
    for M in (1, 8):
        acc = bl.bl_zero_gemm(to_dev(np.repeat(a, M, 0)), to_dev(oracle.pack_ternary(w)))
        assert np.all(acc.cpu().numpy() == -149)


@pytest.mark.parametrize("M,K,N", [(256, 4096, 2048), (300, 2560, 640)])
def test_zero_gemm_split_k(bl, M, K, N):
    """Few output tiles: the tensor-core launch splits K into ranges whose INT32
    partials a second pass sums; results must stay exact, also when M is not a
    multiple of the token tile (300: the last tile's rows past M must not
    reach the next range's partials)."""
    Aq = random_int8(M, K, seed=M + 11)
    codes = random_codes(N, K, seed=N + 13)
    acc = bl.bl_zero_gemm(to_dev(Aq), to_dev(oracle.pack_ternary(codes))).cpu().numpy()
    np.testing.assert_array_equal(acc, oracle.zero_gemm(Aq, codes))
    # twice in a row: the arrival counters must be ready for the next launch
    acc2 = bl.bl_zero_gemm(to_dev(Aq), to_dev(oracle.pack_ternary(codes))).cpu().numpy()
    np.testing.assert_array_equal(acc2, acc)


def test_linear_split_k_down_projection_shape(bl):
    """512 tokens, K = 11008 → N = 4096 (the FFN down-projection's shape: 64
    tiles, so K is split); sampled tokens × rows against the oracle."""
    M, K, N = 512, 11008, 4096
    _linear_case(bl, M, K, N, "bf16", "bf16", True, torch.bfloat16, seed=2,
                 tok=[0, 1, 255, 256, 511], rows=list(range(0, 130)) + list(range(3990, 4096)))


def test_zero_gemm_prefill_sampled(bl):
    """Full prefill size (2048 × 4096 × 4096) in the launch the benchmark
    uses; sampled tokens × rows checked against the oracle."""
    M, K, N = 2048, 4096, 4096
    Aq = random_int8(M, K, seed=3)
    codes = random_codes(N, K, seed=4)
    acc = bl.bl_zero_gemm(to_dev(Aq), to_dev(oracle.pack_ternary(codes))).cpu().numpy()
    tok = np.array([0, 1, 255, 256, 1000, 2047])
    rows = np.concatenate([np.arange(0, 130), np.arange(3967, 4096), [2048, 2049]])
    ref = oracle.zero_gemm(Aq[tok], codes[rows])
    np.testing.assert_array_equal(acc[np.ix_(tok, rows)], ref)


# ---------------------------------------------------------------------------
# a2 + a3 + a4: BitLinear forward

def _linear_case(bl, M, K, N, w_dt, a_dt, outl, out_dtype, relu2=False, seed=0,
                 tok=None, rows=None, pdl=False):
    W = si.weights(N, K, seed=seed, dtype=w_dt)
    codes, g = oracle.quant_weights(W.f32, EPS)
    packed = to_dev(oracle.pack_ternary(codes))
    gamma = to_dev(np.array([g], np.float32))
    A = si.activations(M, K, seed=seed, outliers=outl, dtype=a_dt)
    Y = bl.bl_linear(A.torch(DEV), packed, gamma, EPS, relu2=relu2, out_dtype=out_dtype, pdl=pdl)
    Y = Y.float().cpu().numpy()
    tok = np.arange(M) if tok is None else np.asarray(tok)
    rows = np.arange(N) if rows is None else np.asarray(rows)
    ref = oracle.bitlinear(A.f32[tok], codes[rows], g, EPS, relu2=relu2)["Y"]
    assert_close(Y[np.ix_(tok, rows)], ref, out_dtype)


def test_linear_single_layer_fp32(bl):
    """Single BitLinear: fp32 W 256×512, 4 tokens, fp32 out."""
    _linear_case(bl, 4, 512, 256, "f32", "f32", False, torch.float32)


@pytest.mark.parametrize("relu2", [False, True])
def test_linear_decode_full(bl, relu2):
    """Decode GEMV: 1 token, K=2560, N=6912, bf16 in/out, outliers."""
    _linear_case(bl, 1, 2560, 6912, "bf16", "bf16", True, torch.bfloat16, relu2=relu2)


def test_linear_decode_pdl(bl):
    _linear_case(bl, 1, 2560, 6912, "bf16", "bf16", True, torch.bfloat16, pdl=True)


@pytest.mark.parametrize("M", [2, 3, 4])
def test_linear_gemv_multi_token(bl, M):
    _linear_case(bl, M, 4096, 1000, "bf16", "bf16", True, torch.bfloat16, seed=M)


def test_linear_small_batch_full(bl):
    """M=16, K=4096, N=11008 (skinny path), all outputs."""
    _linear_case(bl, 16, 4096, 11008, "bf16", "bf16", True, torch.bfloat16)


def test_linear_prefill_sampled(bl):
    """M=2048, K=4096, N=4096 bf16: sampled tokens and rows."""
    _linear_case(bl, 2048, 4096, 4096, "bf16", "bf16", True, torch.bfloat16,
                 tok=[0, 5, 255, 256, 1023, 1500, 2047],
                 rows=list(range(0, 160)) + list(range(4000, 4096)))


@pytest.mark.parametrize("M,K,N", [(5, 192, 200), (37, 512, 300), (200, 320, 128), (64, 2560, 512),
                                   (330, 256, 9000), (400, 256, 11008)])
@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16])
def test_linear_ragged(bl, M, K, N, out):
    _linear_case(bl, M, K, N, "f32", "f32", True, out, relu2=(M % 2 == 1))


@pytest.mark.parametrize("M", [3, 48])
def test_linear_q_parity(bl, M):
    K, N = 512, 384
    W = si.weights(N, K, seed=9)
    codes, g = oracle.quant_weights(W.f32, EPS)
    A = si.activations(M, K, seed=9)
    Aq, gA = oracle.quant_acts(A.f32, EPS)
    args = (to_dev(Aq), to_dev(gA), to_dev(oracle.pack_ternary(codes)), to_dev(np.array([g], np.float32)))
    ref = oracle.dequant(oracle.zero_gemm(Aq, codes), gA, g)
    Y1 = bl.bl_linear_q(*args, out_dtype=torch.float32).cpu().numpy()
    rs = to_dev(Aq.astype(np.int32).sum(axis=1).astype(np.int32))
    Y2 = bl.bl_linear_q(*args, rowsum=rs, out_dtype=torch.float32).cpu().numpy()
    assert_close(Y1, ref, torch.float32)
    assert_close(Y2, ref, torch.float32)


# ---------------------------------------------------------------------------
# a5: ternary FFN block

def _ffn_case(bl, M, K, H, seed=0, tok=None, rows=None):
    Wu = si.weights(H, K, seed=seed + 1, dtype="bf16")
    Wd = si.weights(K, H, seed=seed + 2, dtype="bf16")
    cu, gu = oracle.quant_weights(Wu.f32, EPS)
    cd, gd = oracle.quant_weights(Wd.f32, EPS)
    X = si.activations(M, K, seed=seed, dtype="bf16")
    Y = bl.bl_ffn_relu2(X.torch(DEV), to_dev(oracle.pack_ternary(cu)), to_dev(np.array([gu], np.float32)),
                        to_dev(oracle.pack_ternary(cd)), to_dev(np.array([gd], np.float32)), EPS)
    Y = Y.float().cpu().numpy()
    tok = np.arange(M) if tok is None else np.asarray(tok)
    rows = np.arange(K) if rows is None else np.asarray(rows)
    o = oracle.ffn_relu2(X.f32[tok], cu, gu, cd[rows], gd, EPS)
    assert_close(Y[np.ix_(tok, rows)], o["Y"], torch.bfloat16)


@pytest.mark.parametrize("M", [1, 2, 4, 5, 17, 64])
def test_ffn_small(bl, M):
    _ffn_case(bl, M, 256, 640, seed=M)


def _random_linear_cases(count, seed):
    u = si.uniform(seed, 5 * count).reshape(count, 5)
    cases = []
    for a, b, c, d, e in u:
        M = int(1 + a ** 3 * 500)
        K = 64 * int(1 + b * 24)
        N = int(8 + c ** 1.5 * 6000)
        out = torch.float32 if d < 0.5 else torch.bfloat16
        cases.append((M, K, N, out, bool(e < 0.3)))
    return cases


@pytest.mark.parametrize("M,K,N,out,relu2", _random_linear_cases(16, seed=77))
def test_linear_random_shapes(bl, M, K, N, out, relu2):
    """Seeded shapes through every dequantising epilogue (GEMV, warp-level,
    tensor-core tiles, K splits), fp32 or bf16 out, ReLU² on some."""
    _linear_case(bl, M, K, N, "bf16", "bf16", True, out, relu2=relu2, seed=M + N)


def _random_ffn_cases(count, seed):
    u = si.uniform(seed, 3 * count).reshape(count, 3)
    return [(int(1 + a ** 2 * 400), 64 * int(2 + b * 14), 64 * int(2 + c * 30)) for a, b, c in u]


@pytest.mark.parametrize("M,K,H", _random_ffn_cases(8, seed=91))
def test_ffn_random_shapes(bl, M, K, H):
    _ffn_case(bl, M, K, H, seed=M + H)


@pytest.mark.parametrize("M", [1, 64, 512])
def test_ffn_full_sampled(bl, M):
    """FFN block 4096 → 11008 → 4096 at M ∈ {1, 64, 512}; sampled tokens."""
    tok = [0] if M == 1 else [0, 1, M // 2, M - 1]
    _ffn_case(bl, M, 4096, 11008, tok=tok)


# ---------------------------------------------------------------------------
# error paths and the bounded-wait machinery

def test_device_error_flag_timeout(bl):
    """A wait that nothing completes gives up after the limit, raises the
    device flag, and the context stays usable."""
    assert bl.bl_check_device_error() == 0
    bl.bl_selftest_wait_timeout(2_000_000)  # 2 ms
    assert bl.bl_check_device_error() == 6  # BL_ERR_TIMEOUT
    assert bl.bl_check_device_error() == 0  # cleared
    x = torch.ones(4, device=DEV)
    assert float(x.sum().item()) == 4.0


def test_argument_errors_launch_nothing(bl):
    A = torch.zeros((4, 100), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(bl.BitLinearError) as e:
        bl.bl_quant_acts(A)
    assert e.value.status == 2
    W = torch.zeros((8, 64), dtype=torch.float16, device=DEV)
    with pytest.raises(TypeError):
        bl.bl_quant_weights(W)


def test_pdl_chain_distinct_weights(bl):
    """A chain of decode calls over distinct weight matrices, launched with
    programmatic dependent launch, gives each layer's own result."""
    K, N = 2560, 1024
    A = si.activations(1, K, seed=0, dtype="bf16")
    At = A.torch(DEV)
    Ws, outs, refs = [], [], []
    for i in range(6):
        W = si.weights(N, K, seed=100 + i, dtype="bf16")
        codes, g = oracle.quant_weights(W.f32, EPS)
        Ws.append((to_dev(oracle.pack_ternary(codes)), to_dev(np.array([g], np.float32))))
        refs.append(oracle.bitlinear(A.f32, codes, g, EPS)["Y"])
    for p, g in Ws:
        outs.append(bl.bl_linear(At, p, g, EPS, pdl=True))
    torch.cuda.synchronize()
    for y, r in zip(outs, refs):
        assert_close(y.float().cpu().numpy(), r, torch.bfloat16)


def test_skinny_chain_shared_workspace(bl):
    """Back-to-back 16-token calls that share one workspace: each call's
    contraction streams its weights before the quantiser of the same call has
    finished (programmatic dependent launch) and must still read its own
    call's tokens, not the next call's."""
    M, K, N = 16, 1024, 2048
    ws = torch.empty(bl.workspace_bytes("linear", M, K, N), dtype=torch.uint8, device=DEV)
    cases, args = [], []
    for i in range(6):
        W = si.weights(N, K, seed=200 + i, dtype="bf16")
        codes, g = oracle.quant_weights(W.f32, EPS)
        A = si.activations(M, K, seed=300 + i, dtype="bf16", outliers=True)
        cases.append((A, codes, g))
        args.append((A.torch(DEV), to_dev(oracle.pack_ternary(codes)),
                     to_dev(np.array([g], np.float32))))
    torch.cuda.synchronize()
    outs = [bl.bl_linear(a, p, g, EPS, workspace=ws) for a, p, g in args]  # back to back
    torch.cuda.synchronize()
    refs = [oracle.bitlinear(A.f32, codes, g, EPS)["Y"] for A, codes, g in cases]
    for y, r in zip(outs, refs):
        assert_close(y.float().cpu().numpy(), r, torch.bfloat16)


@pytest.mark.parametrize("M", [16, 20, 40])
def test_small_batch_pdl_chain_shared_workspace(bl, M):
    """Chained calls with programmatic dependent launch sharing one workspace:
    each call's quantiser launches early but must wait for the previous call
    before overwriting the shared int8 tokens, and the contraction streams its
    weights before it waits for the quantiser. Every call must give its own
    result."""
    K, N = 4096, 3000
    ws = torch.empty(bl.workspace_bytes("linear", M, K, N), dtype=torch.uint8, device=DEV)
    cases, args = [], []
    for i in range(6):
        W = si.weights(N, K, seed=500 + i, dtype="bf16")
        codes, g = oracle.quant_weights(W.f32, EPS)
        A = si.activations(M, K, seed=600 + i, dtype="bf16", outliers=True)
        cases.append((A, codes, g))
        args.append((A.torch(DEV), to_dev(oracle.pack_ternary(codes)),
                     to_dev(np.array([g], np.float32))))
    torch.cuda.synchronize()
    outs = [bl.bl_linear(a, p, g, EPS, workspace=ws, pdl=True) for a, p, g in args]
    torch.cuda.synchronize()
    for (A, codes, g), y in zip(cases, outs):
        assert_close(y.float().cpu().numpy(), oracle.bitlinear(A.f32, codes, g, EPS)["Y"], torch.bfloat16)


@pytest.mark.parametrize("M", [1, 16, 130])
def test_ffn_pdl_chain_shared_workspace(bl, M):
    """Chained FFN blocks with programmatic dependent launch on one shared
    workspace: the next block's first kernel starts early but must not touch
    the workspace or read its input before the previous block is done."""
    K, H = 1024, 2752
    ws = torch.empty(bl.workspace_bytes("ffn", M, K, H), dtype=torch.uint8, device=DEV)
    blocks = []
    for i in range(4):
        cu, gu = oracle.quant_weights(si.weights(H, K, seed=700 + i, dtype="bf16").f32, EPS)
        cd, gd = oracle.quant_weights(si.weights(K, H, seed=800 + i, dtype="bf16").f32, EPS)
        X = si.activations(M, K, seed=900 + i, dtype="bf16", outliers=True)
        blocks.append((X, cu, gu, cd, gd))
    dev = [(X.torch(DEV), to_dev(oracle.pack_ternary(cu)), to_dev(np.array([gu], np.float32)),
            to_dev(oracle.pack_ternary(cd)), to_dev(np.array([gd], np.float32)))
           for X, cu, gu, cd, gd in blocks]
    torch.cuda.synchronize()
    outs = [bl.bl_ffn_relu2(*d, EPS, workspace=ws, pdl=True) for d in dev]
    torch.cuda.synchronize()
    for (X, cu, gu, cd, gd), y in zip(blocks, outs):
        assert_close(y.float().cpu().numpy(), oracle.ffn_relu2(X.f32, cu, gu, cd, gd, EPS)["Y"],
                     torch.bfloat16)


def test_mixed_pdl_chain_shared_workspace(bl):
    """Calls of every contraction path (GEMV, warp-level MMA, tensor-core tiles
    with and without K split) and FFN blocks, chained with programmatic
    dependent launch on one stream and one shared workspace. Each kernel may
    start before its predecessor ends, so one that read its inputs or reused
    the shared scratch too early would change a result: every output must
    equal the same call made alone, bit for bit."""
    K, N, H = 1024, 1536, 2048
    W = si.weights(N, K, seed=41, dtype="bf16").torch(DEV)
    Wu = si.weights(H, K, seed=42, dtype="bf16").torch(DEV)
    Wd = si.weights(K, H, seed=43, dtype="bf16").torch(DEV)
    pw, gw = bl.bl_quant_weights(W, EPS)
    pu, gu = bl.bl_quant_weights(Wu, EPS)
    pd, gd = bl.bl_quant_weights(Wd, EPS)
    seq = [("linear", 1), ("linear", 16), ("ffn", 64), ("linear", 200), ("ffn", 1),
           ("linear", 40), ("ffn", 300), ("linear", 3), ("linear", 600), ("ffn", 16),
           ("linear", 64), ("ffn", 4)]
    need = max(bl.workspace_bytes("linear" if op == "linear" else "ffn", M, K,
                                  N if op == "linear" else H) for op, M in seq)
    ws = torch.empty(max(1, need), dtype=torch.uint8, device=DEV)
    xs = [si.activations(M, K, seed=1000 + i, dtype="bf16", outliers=True).torch(DEV)
          for i, (_, M) in enumerate(seq)]

    def call(i, pdl, workspace):
        op, M = seq[i]
        if op == "linear":
            return bl.bl_linear(xs[i], pw, gw, EPS, workspace=workspace, pdl=pdl)
        return bl.bl_ffn_relu2(xs[i], pu, gu, pd, gd, EPS, workspace=workspace, pdl=pdl)

    torch.cuda.synchronize()
    alone = []
    for i in range(len(seq)):
        alone.append(call(i, False, None))
        torch.cuda.synchronize()
    for _ in range(2):
        chained = [call(i, True, ws) for i in range(len(seq))]
        torch.cuda.synchronize()
        for i, (y, r) in enumerate(zip(chained, alone)):
            assert torch.equal(y, r), f"call {i} {seq[i]} differs when chained"
    assert bl.bl_check_device_error() == 0


@pytest.mark.parametrize("M", [1, 2, 16, 100])
def test_wide_output_sampled(bl, M):
    """An output as wide as a language-model head (128,256 rows × 2048
    inputs): every path runs several waves of CTAs over the SMs (GEMV slabs,
    128-row warp-level slabs, 128-row tensor-core tiles). The matrix repeats
    one seeded 8192-row block; sampled rows from different repeats, the first
    and the last are checked bit-exactly against the oracle."""
    K, N = 2048, 128256
    codes = np.tile(random_codes(8192, K, seed=99), (N // 8192 + 1, 1))[:N]
    packed = to_dev(oracle.pack_ternary(codes))
    Aq = random_int8(M, K, seed=500 + M)
    acc = bl.bl_zero_gemm(to_dev(Aq), packed).cpu().numpy()
    rows = [0, 1, 127, 128, 8191, 8192, 65535, 65536, 100000, 128127, N - 2, N - 1]
    np.testing.assert_array_equal(acc[:, rows], oracle.zero_gemm(Aq, np.ascontiguousarray(codes[rows])))
