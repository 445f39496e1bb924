"""GPU parity of the FP8 weight tier against the oracle.

The tier stores W as E4M3 codes [N][K] with one fp32 scale per row (reading
R15: s_n = amax|W[n]| / 448, code = E4M3_RNE_satfinite(w / s_n)); the GPU
quantiser must reproduce the oracle's codes and scales bit for bit, and the
linear must meet the stated tolerance against the oracle's fp64 sum of
e4m3(code) * s_n * x. Runs on the MMA variant (the default, every M) and on
the row-block variant (forced, M <= 2).
"""
import numpy as np
import pytest
import torch

import nvfp4_weight_streaming_b200 as nv
import oracle
import synth
from tests.gpu_util import Guarded, check_tolerance, dev, host_u16

pytestmark = pytest.mark.gpu


def gpu_quantize_fp8(W):
    N, K = W.shape
    wd = torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda()
    codes = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
    sc = torch.zeros(N, dtype=torch.float32, device="cuda")
    bad = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_quantize_fp8(wd, N, K, codes, sc, bad)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), sc.cpu().numpy(), int(bad.item())


def fp8_cases():
    rng = np.random.default_rng(5)
    yield synth.normal_f32(64 * 512, 0.02, seed=1, stream=7).reshape(64, 512)
    W = (np.exp2(rng.uniform(-40, 8, (32, 256))) * rng.choice([-1, 1], (32, 256))).astype(np.float32)
    yield W
    W = rng.normal(0, 1, (16, 128)).astype(np.float32)
    W[2] = 0.0                                  # zero row: scale 0, zero codes
    W[5, 3] = -1e-30                            # rounds to -0: code 0x80
    W[5, 4] = 1e-30
    W[7] = np.float32(448.0)                    # scale 1, all codes 0x7E
    yield W


@pytest.mark.parametrize("case", range(3))
def test_fp8_quantizer_bit_exact(case):
    W = list(fp8_cases())[case]
    codes, sc, bad = gpu_quantize_fp8(W)
    rc, rs = oracle.quantize_fp8_rows(W)
    assert bad == 0
    assert np.array_equal(sc.view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(codes, rc)


def test_fp8_quantizer_flags_nonfinite():
    W = np.ones((2, 32), np.float32)
    W[0, 3] = np.nan
    W[1, 9] = np.inf
    assert gpu_quantize_fp8(W)[2] == 2


def run_fp8(codes, sc, X, gs=1.0, repeat=1, variant=0):
    M, K = X.shape
    N = codes.shape[0]
    plan = nv.nvfp4_linear_plan(M, N, K, torch.cuda.current_device(), nv.NVFP4_PLAN_WEIGHT_FP8 | variant)
    try:
        assert nv.nvfp4_linear_variant(plan) == (variant or nv.NVFP4_VARIANT_MMA)
        wsb = nv.nvfp4_linear_workspace_bytes(plan)
        ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
        cd = torch.from_numpy(codes).cuda()
        sd = torch.from_numpy(sc).cuda()
        gd = torch.tensor([gs], dtype=torch.float32, device="cuda")
        y = Guarded(M * N)
        xd = dev(X)
        for _ in range(repeat):
            nv.nvfp4_linear_run(plan, cd, sd, gd, xd, y.view, ws, wsb)
        assert nv.nvfp4_linear_status(plan, ws) == nv.NVFP4_OK
        assert y.guards_intact()
        return host_u16(y.view).reshape(M, N)
    finally:
        nv.nvfp4_linear_destroy(plan)


@pytest.mark.parametrize("M,N,K", [(1, 520, 512), (2, 1000, 768), (1, 2, 256), (2, 2339, 5120),
                                   (1, 34816, 5120), (1, 5120, 17408), (3, 777, 1280),
                                   (4, 130 * 256 - 77, 512),
                                   # X in the ring (M >= 5)
                                   (5, 129, 256), (8, 2339, 1280), (16, 34816, 5120), (16, 5120, 17408)])
@pytest.mark.parametrize("variant", [0, nv.NVFP4_VARIANT_ROW])
def test_fp8_linear(M, N, K, variant):
    if variant == nv.NVFP4_VARIANT_ROW and M > 2:
        pytest.skip("the row variant takes M <= 2")
    W = synth.normal_f32(N * K, 0.02, seed=N + K, stream=7).reshape(N, K)
    codes, sc = oracle.quantize_fp8_rows(W)
    X = synth.x_bf16_custom(synth.X_OUTLIERS, M, K, seed=K, n_outliers=8, gain=20.0)
    y = run_fp8(codes, sc, X, variant=variant)
    y_ref, ad = oracle.linear_fp8(codes, sc, X, M, N, K)
    check_tolerance(y, y_ref, ad)


def test_fp8_dyadic_case_is_exact_on_both_variants():
    """Integer weights |v| <= 8 (exact E4M3 codes, from torch's conversion),
    unit row scales and integer X: every partial sum is an exact integer in
    fp32, so both variants must return the oracle's value rounded to bf16."""
    M, N, K = 2, 300, 512
    rng = np.random.default_rng(11)
    vals = rng.integers(-8, 9, size=(N, K)).astype(np.float32)
    codes = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    sc = np.ones(N, np.float32)
    X = oracle.bf16_round_array(rng.integers(-4, 5, size=(M, K)).astype(np.float64))
    y_ref, _ = oracle.linear_fp8(codes, sc, X, M, N, K)
    want = oracle.bf16_bits_to_f64(oracle.bf16_round_array(y_ref))
    for variant in (0, nv.NVFP4_VARIANT_ROW):
        got = oracle.bf16_bits_to_f64(run_fp8(codes, sc, X, variant=variant))
        assert np.array_equal(got, want), variant


def test_fp8_linear_global_scale_multiplies():
    """w_global multiplies every weight: gs = 2 doubles Y exactly."""
    M, N, K = 2, 777, 1024
    W = synth.normal_f32(N * K, 0.02, seed=3, stream=7).reshape(N, K)
    codes, sc = oracle.quantize_fp8_rows(W)
    X = synth.x_bf16_custom(synth.X_NORMAL, M, K, seed=4)
    y1 = oracle.bf16_bits_to_f64(run_fp8(codes, sc, X, 1.0))
    y2 = oracle.bf16_bits_to_f64(run_fp8(codes, sc, X, 2.0))
    assert np.array_equal(2 * y1, y2)


def test_fp8_wide_x_uses_the_lo_plane():
    M, N, K = 2, 1031, 5120
    rng = np.random.default_rng(8)
    big = np.sort(rng.choice(K, 6, replace=False))
    W = synth.normal_f32(N * K, 0.02, seed=9, stream=7).reshape(N, K)
    W[:, big] = 0.0
    codes, sc = oracle.quantize_fp8_rows(W)
    X = synth.x_bf16_custom(synth.X_NORMAL, M, K, seed=10)
    mant = rng.uniform(1.0, 2.0, K)
    x = rng.choice([-1.0, 1.0], K) * mant * np.exp2(rng.integers(-15, -5, K).astype(np.float64))
    x[big] = 2.0 ** 40
    X[1] = oracle.bf16_round_array(x)
    y = run_fp8(codes, sc, X)
    y_ref, ad = oracle.linear_fp8(codes, sc, X, M, N, K)
    tol = oracle.tolerance(y_ref, ad)
    assert np.mean(np.abs(y_ref[1]) > tol[1]) > 0.95
    check_tolerance(y, y_ref, ad)


def test_fp8_deterministic():
    M, N, K = 1, 34816, 5120
    W = synth.normal_f32(N * K, 0.02, seed=N + K, stream=7).reshape(N, K)
    codes, sc = oracle.quantize_fp8_rows(W)
    X = synth.x_bf16_custom(synth.X_NORMAL, M, K, seed=2)
    assert np.array_equal(run_fp8(codes, sc, X), run_fp8(codes, sc, X, repeat=3))


def test_fp8_plan_limits():
    d = torch.cuda.current_device()
    for flags in (nv.NVFP4_PLAN_WEIGHT_FP8 | nv.NVFP4_VARIANT_GEMV,
                  nv.NVFP4_PLAN_WEIGHT_FP8 | nv.NVFP4_VARIANT_TC,
                  nv.NVFP4_PLAN_WEIGHT_FP8 | nv.NVFP4_PLAN_EPI_SWIGLU,
                  nv.NVFP4_PLAN_WEIGHT_FP8 | nv.NVFP4_PLAN_ACT_NVFP4):
        with pytest.raises(nv.Nvfp4Error) as e:
            nv.nvfp4_linear_plan(1, 1024, 512, d, flags)
        assert e.value.status == nv.NVFP4_ERR_UNSUPPORTED
    for M, flags in ((5, nv.NVFP4_VARIANT_ROW), (3, nv.NVFP4_VARIANT_ROW)):
        with pytest.raises(nv.Nvfp4Error) as e:
            nv.nvfp4_linear_plan(M, 1024, 512, d, nv.NVFP4_PLAN_WEIGHT_FP8 | flags)
        assert e.value.status == nv.NVFP4_ERR_UNSUPPORTED
    for M in (4, 16):
        p = nv.nvfp4_linear_plan(M, 1024, 512, d, nv.NVFP4_PLAN_WEIGHT_FP8)
        try:
            assert nv.nvfp4_linear_variant(p) == nv.NVFP4_VARIANT_MMA
        finally:
            nv.nvfp4_linear_destroy(p)
