"""GPU parity of the W4A4 tier against the oracle.

The plan flag NVFP4_PLAN_ACT_NVFP4 quantises X to NVFP4 on the GPU (reading
R14: 16-element blocks of a token row, E4M3 block scales, per-tensor scale
amax(|X|)/(6*448) of the call's X, the weights' quantiser steps). Two
variants take it: MMA (codes decoded to f16 for the warp MMA) and TC (the
block-scaled FP4 tensor cores, tcgen05.mma kind::mxf4nvf4, no decode). Both
must meet the stated tolerance against the oracle's fp64 sum of
w_hat * x_hat, with x_hat from the oracle's own activation quantiser.
"""
import numpy as np
import pytest
import torch

import nvfp4_weight_streaming_b200 as nv
import oracle
import synth
from tests.gpu_util import Guarded, Weights, check_tolerance, dev, host_u16

pytestmark = pytest.mark.gpu


VARIANTS = [nv.NVFP4_VARIANT_MMA, nv.NVFP4_VARIANT_TC]


def run_w4a4(w, X, flags=0, variant=nv.NVFP4_VARIANT_MMA):
    """Y bits [M][N] of the W4A4 linear through the C ABI."""
    M, K = X.shape
    plan = nv.nvfp4_linear_plan(M, w.N, K, torch.cuda.current_device(),
                                nv.NVFP4_PLAN_ACT_NVFP4 | variant | flags)
    try:
        assert nv.nvfp4_linear_variant(plan) == variant
        wsb = nv.nvfp4_linear_workspace_bytes(plan)
        ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
        y = Guarded(M * w.N)
        nv.nvfp4_linear_run(plan, w.packed, w.scales, w.gsd, dev(X), y.view, ws if wsb else None, wsb)
        assert nv.nvfp4_linear_status(plan, ws if wsb else None) == nv.NVFP4_OK
        assert y.guards_intact()
        return host_u16(y.view).reshape(M, w.N)
    finally:
        nv.nvfp4_linear_destroy(plan)


def reference(w, X):
    M, K = X.shape
    xp, xs, gsx = oracle.quantize_x(X)
    return oracle.linear_w4a4(w.packed_h, w.scales_h, w.gs, xp, xs, gsx, M, w.N, K)


def weights(N, K, seed):
    W = synth.normal_f32(N * K, 0.02, seed=seed, stream=7).reshape(N, K)
    return Weights(*oracle.quantize(W))


SHAPES = [(1, 520, 512), (2, 1000, 768), (3, 777, 1280), (4, 4097, 512),
          (1, 130 * 256 - 77, 512), (1, 34816, 5120), (2, 34816, 5120),
          (1, 5120, 17408),
          (4, 1024, 17408),      # MMA: X in K-slices, each CTA quantises its slice; TC: K split 37 ways
          # MMA, M >= 5: X in the ring, quantised by the X-conversion kernel
          (5, 129, 256), (8, 2339, 1280), (16, 34816, 5120), (16, 5120, 17408),
          # TC: more tiles than SMs (CTAs loop over tiles, double-buffered accumulators)
          (3, 300 * 256 - 5, 512), (16, 160 * 256, 256),
          # TC: one K-step (fewer steps than ring stages), K split over few steps
          (7, 4096, 256), (12, 4096, 4096)]


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_w4a4_linear(M, N, K, variant):
    w = weights(N, K, seed=N + K)
    X = synth.x_bf16_custom(synth.X_OUTLIERS, M, K, seed=K + M, n_outliers=8, gain=20.0)
    y = run_w4a4(w, X, variant=variant)
    y_ref, ad = reference(w, X)
    check_tolerance(y, y_ref, ad)


@pytest.mark.parametrize("M,N,K", [(1, 5120, 17408), (16, 34816, 5120), (5, 300 * 256, 512)])
def test_w4a4_tc_repeats_bit_for_bit(M, N, K):
    """Split-K sums run in slice order, whole tiles in K order: two calls on
    the same inputs give the same bits (and so does a third after other X)."""
    w = weights(N, K, seed=3)
    X = synth.x_bf16_custom(synth.X_NORMAL, M, K, seed=11)
    X2 = synth.x_bf16_custom(synth.X_NORMAL, M, K, seed=12)
    a = run_w4a4(w, X, variant=nv.NVFP4_VARIANT_TC)
    run_w4a4(w, X2, variant=nv.NVFP4_VARIANT_TC)
    b = run_w4a4(w, X, variant=nv.NVFP4_VARIANT_TC)
    assert np.array_equal(a, b)


def test_w4a4_tc_plan_shape():
    """Three launches (X amax, X quantisation, the stream); K split only when
    the tiles leave SMs idle."""
    d = torch.cuda.current_device()
    for M, N, K, split in [(1, 34816, 5120, False), (16, 248320, 5120, False), (1, 5120, 17408, True)]:
        p = nv.nvfp4_linear_plan(M, N, K, d, nv.NVFP4_PLAN_ACT_NVFP4 | nv.NVFP4_VARIANT_TC)
        try:
            assert nv.nvfp4_linear_launches_per_run(p) == 3
            assert (nv.nvfp4_linear_split_k(p) > 1) == split
        finally:
            nv.nvfp4_linear_destroy(p)


def test_w4a4_tc_forced_timeout_reports_status_and_recovers():
    """Test-only flag: the producer issues nothing, the MMA warp's bounded wait
    runs out, the kernel reports NVFP4_ERR_TIMEOUT and returns; the workspace,
    cleared by the status call, then serves a normal run."""
    M, N, K = 2, 1000, 768
    w = weights(N, K, seed=5)
    X = synth.x_bf16_custom(synth.X_NORMAL, M, K, seed=5)
    d = torch.cuda.current_device()
    plan = nv.nvfp4_linear_plan(M, N, K, d, nv.NVFP4_PLAN_ACT_NVFP4 | nv.NVFP4_VARIANT_TC |
                                nv.NVFP4_PLAN_TEST_STALL)
    try:
        wsb = nv.nvfp4_linear_workspace_bytes(plan)
        ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
        y = Guarded(M * N)
        nv.nvfp4_linear_run(plan, w.packed, w.scales, w.gsd, dev(X), y.view, ws, wsb)
        assert nv.nvfp4_linear_status(plan, ws) == nv.NVFP4_ERR_TIMEOUT
        assert y.guards_intact()
        assert int(ws.sum()) == 0
    finally:
        nv.nvfp4_linear_destroy(plan)
    y_ref, ad = reference(w, X)
    check_tolerance(run_w4a4(w, X, variant=nv.NVFP4_VARIANT_TC), y_ref, ad)


@pytest.mark.parametrize("variant", VARIANTS)
def test_w4a4_differs_from_the_bf16_linear_as_the_oracle_does(variant):
    """The tier changes the numerics: on X with a wide spread the quantised
    product is measurably different from the W4A16 one, and the GPU follows
    the W4A4 reference, not the bf16 one."""
    M, N, K = 1, 2048, 1024
    w = weights(N, K, seed=4)
    X = synth.x_bf16_custom(synth.X_OUTLIERS, M, K, seed=9, n_outliers=8, gain=20.0)
    y = oracle.bf16_bits_to_f64(run_w4a4(w, X, variant=variant))
    y4, ad4 = reference(w, X)
    y16, _ = oracle.linear(w.packed_h, w.scales_h, w.gs, X, M, N, K)
    err4 = np.abs(y - y4).max()
    err16 = np.abs(y - y16).max()
    assert err16 > 10 * err4


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("M", [2, 12])
def test_w4a4_doubling_x_doubles_y_exactly(M, variant):
    N, K = 777, 1024
    w = weights(N, K, seed=6)
    X = synth.x_bf16_custom(synth.X_NORMAL, M, K, seed=7)
    X2 = oracle.bf16_round_array(2.0 * oracle.bf16_bits_to_f64(X))
    y1 = oracle.bf16_bits_to_f64(run_w4a4(w, X, variant=variant))
    y2 = oracle.bf16_bits_to_f64(run_w4a4(w, X2, variant=variant))
    assert np.array_equal(2 * y1, y2)


@pytest.mark.parametrize("variant", VARIANTS)
def test_w4a4_zero_x_gives_zero_y_and_repeats(variant):
    M, N, K = 1, 1000, 512
    w = weights(N, K, seed=8)
    X = np.zeros((M, K), np.uint16)
    assert not run_w4a4(w, X, variant=variant).any()
    X = synth.x_bf16_custom(synth.X_NORMAL, M, K, seed=8)
    assert np.array_equal(run_w4a4(w, X, variant=variant), run_w4a4(w, X, variant=variant))


def test_w4a4_variants_agree_closely():
    """Both variants quantise X the same way (bit-identical codes and scales),
    so their outputs differ only by fp32 summation order."""
    M, N, K = 4, 4096, 5120
    w = weights(N, K, seed=9)
    X = synth.x_bf16_custom(synth.X_OUTLIERS, M, K, seed=9, n_outliers=8, gain=20.0)
    a = oracle.bf16_bits_to_f64(run_w4a4(w, X, variant=nv.NVFP4_VARIANT_MMA))
    b = oracle.bf16_bits_to_f64(run_w4a4(w, X, variant=nv.NVFP4_VARIANT_TC))
    _, ad = reference(w, X)
    # at most one bf16 rounding step apart, and that only where the fp32 sums
    # straddle a rounding boundary
    d = np.abs(a - b)
    assert np.all(d <= 2.0 ** -7 * np.maximum(np.abs(a), np.abs(b)) + 1e-5 * ad)
    assert np.count_nonzero(d) <= 0.05 * d.size


def test_w4a4_plan_limits():
    d = torch.cuda.current_device()
    bad = [(1, 1024, 512, nv.NVFP4_VARIANT_GEMV), (1, 1024, 512, nv.NVFP4_VARIANT_ROW),
           (1, 1024, 512, nv.NVFP4_PLAN_WEIGHT_FP8),
           (1, 1024, 512, nv.NVFP4_VARIANT_TC | nv.NVFP4_PLAN_EPI_SWIGLU)]
    for M, N, K, flags in bad:
        with pytest.raises(nv.Nvfp4Error) as e:
            nv.nvfp4_linear_plan(M, N, K, d, nv.NVFP4_PLAN_ACT_NVFP4 | flags)
        assert e.value.status == nv.NVFP4_ERR_UNSUPPORTED, (M, N, K, flags)


def test_w4a4_auto_choice():
    """AUTO: the FP4 tensor cores from M = 4 on, the warp-MMA kernel below that
    and for the fused epilogues."""
    d = torch.cuda.current_device()
    for M, flags, want in [(1, 0, nv.NVFP4_VARIANT_MMA), (3, 0, nv.NVFP4_VARIANT_MMA),
                           (4, 0, nv.NVFP4_VARIANT_TC), (16, 0, nv.NVFP4_VARIANT_TC),
                           (16, nv.NVFP4_PLAN_EPI_SWIGLU, nv.NVFP4_VARIANT_MMA),
                           (8, nv.NVFP4_PLAN_EPI_ARGMAX, nv.NVFP4_VARIANT_MMA)]:
        p = nv.nvfp4_linear_plan(M, 2048, 1024, d, nv.NVFP4_PLAN_ACT_NVFP4 | flags)
        try:
            assert nv.nvfp4_linear_variant(p) == want, (M, flags)
        finally:
            nv.nvfp4_linear_destroy(p)


def _run_epi(w, X, flags, count):
    M, K = X.shape
    plan = nv.nvfp4_linear_plan(M, w.N, K, torch.cuda.current_device(), nv.NVFP4_PLAN_ACT_NVFP4 | flags)
    try:
        assert nv.nvfp4_linear_variant(plan) == nv.NVFP4_VARIANT_MMA
        wsb = nv.nvfp4_linear_workspace_bytes(plan)
        ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
        y = Guarded(count)
        nv.nvfp4_linear_run(plan, w.packed, w.scales, w.gsd, dev(X), y.view, ws, wsb)
        assert nv.nvfp4_linear_status(plan, ws) == nv.NVFP4_OK
        assert y.guards_intact()
        return y.view.cpu().numpy()
    finally:
        nv.nvfp4_linear_destroy(plan)


@pytest.mark.parametrize("M", [1, 5, 16])
def test_w4a4_swiglu_epilogue(M):
    """W4A4 with the fused SwiGLU epilogue: silu(gate) * up of the quantised
    product, within the SwiGLU bound built from the W4A4 reference."""
    N, K = 2 * 777, 1280
    w = weights(N, K, seed=21)
    X = synth.x_bf16_custom(synth.X_OUTLIERS, M, K, seed=22, n_outliers=4, gain=20.0)
    got = oracle.bf16_bits_to_f64(_run_epi(w, X, nv.NVFP4_PLAN_EPI_SWIGLU, M * (N // 2)).view(np.uint16)
                                  .reshape(M, N // 2))
    y4, ad4 = reference(w, X)
    g, u = y4[:, 0::2], y4[:, 1::2]
    h = np.vectorize(oracle.silu, otypes=[np.float64])(g) * u
    tol = oracle.swiglu_tolerance(h, g, u, ad4[:, 0::2], ad4[:, 1::2])
    assert np.all(np.abs(got - h) <= tol)


@pytest.mark.parametrize("M", [1, 5, 16])
def test_w4a4_argmax_epilogue(M):
    """W4A4 with the fused argmax: the W4A4 reference's top row wherever the
    top-2 gap exceeds the two logits' bounds, else a row within them; the
    reported value within its logit's bound."""
    N, K = 5000, 1024
    w = weights(N, K, seed=23)
    X = synth.x_bf16_custom(synth.X_NORMAL, M, K, seed=24)
    out = _run_epi(w, X, nv.NVFP4_PLAN_EPI_ARGMAX, 4 * M).view(np.uint8)
    idx = out[:4 * M].view(np.int32)
    val = out[4 * M:].view(np.float32).astype(np.float64)
    y4, ad4 = reference(w, X)
    tol = oracle.tolerance(y4, ad4)
    top, decided = oracle.argmax_decided(y4, tol)
    for m in range(M):
        j = int(idx[m])
        assert 0 <= j < N
        if decided[m]:
            assert j == top[m], (m, j, int(top[m]))
        else:
            assert y4[m, top[m]] - y4[m, j] <= tol[m, top[m]] + tol[m, j]
        assert abs(val[m] - y4[m, j]) <= tol[m, j]
