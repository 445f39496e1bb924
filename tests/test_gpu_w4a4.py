"""GPU parity of the W4A4 tier against the oracle.

The plan flag NVFP4_PLAN_ACT_NVFP4 makes the MMA kernel quantise X to NVFP4
itself (reading R14: 16-element blocks of a token row, E4M3 block scales,
per-tensor scale amax(|X|)/(6*448) of the call's X, the weights' quantiser
steps). The result must meet the stated tolerance against the oracle's fp64
sum of w_hat * x_hat, with x_hat from the oracle's own activation quantiser.
"""
import numpy as np
import pytest
import torch

import nvfp4_weight_streaming_b200 as nv
import oracle
import synth
from tests.gpu_util import Guarded, Weights, check_tolerance, dev, host_u16

pytestmark = pytest.mark.gpu


def run_w4a4(w, X, flags=0):
    """Y bits [M][N] of the W4A4 linear through the C ABI (MMA variant)."""
    M, K = X.shape
    plan = nv.nvfp4_linear_plan(M, w.N, K, torch.cuda.current_device(), nv.NVFP4_PLAN_ACT_NVFP4 | flags)
    try:
        assert nv.nvfp4_linear_variant(plan) == nv.NVFP4_VARIANT_MMA
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


@pytest.mark.parametrize("M,N,K", [(1, 520, 512), (2, 1000, 768), (3, 777, 1280), (4, 4097, 512),
                                   (1, 130 * 256 - 77, 512), (1, 34816, 5120), (2, 34816, 5120),
                                   (1, 5120, 17408),
                                   (4, 1024, 17408),      # X in K-slices: each CTA quantises its slice
                                   # M >= 5: X in the ring, quantised by the X-conversion kernel
                                   (5, 129, 256), (8, 2339, 1280), (16, 34816, 5120), (16, 5120, 17408)])
def test_w4a4_linear(M, N, K):
    w = weights(N, K, seed=N + K)
    X = synth.x_bf16_custom(synth.X_OUTLIERS, M, K, seed=K + M, n_outliers=8, gain=20.0)
    y = run_w4a4(w, X)
    y_ref, ad = reference(w, X)
    check_tolerance(y, y_ref, ad)


def test_w4a4_differs_from_the_bf16_linear_as_the_oracle_does():
    """The tier changes the numerics: on X with a wide spread the quantised
    product is measurably different from the W4A16 one, and the GPU follows
    the W4A4 reference, not the bf16 one."""
    M, N, K = 1, 2048, 1024
    w = weights(N, K, seed=4)
    X = synth.x_bf16_custom(synth.X_OUTLIERS, M, K, seed=9, n_outliers=8, gain=20.0)
    y = oracle.bf16_bits_to_f64(run_w4a4(w, X))
    y4, ad4 = reference(w, X)
    y16, _ = oracle.linear(w.packed_h, w.scales_h, w.gs, X, M, N, K)
    err4 = np.abs(y - y4).max()
    err16 = np.abs(y - y16).max()
    assert err16 > 10 * err4


@pytest.mark.parametrize("M", [2, 12])
def test_w4a4_doubling_x_doubles_y_exactly(M):
    N, K = 777, 1024
    w = weights(N, K, seed=6)
    X = synth.x_bf16_custom(synth.X_NORMAL, M, K, seed=7)
    X2 = oracle.bf16_round_array(2.0 * oracle.bf16_bits_to_f64(X))
    y1 = oracle.bf16_bits_to_f64(run_w4a4(w, X))
    y2 = oracle.bf16_bits_to_f64(run_w4a4(w, X2))
    assert np.array_equal(2 * y1, y2)


def test_w4a4_zero_x_gives_zero_y_and_repeats():
    M, N, K = 1, 1000, 512
    w = weights(N, K, seed=8)
    X = np.zeros((M, K), np.uint16)
    assert not run_w4a4(w, X).any()
    X = synth.x_bf16_custom(synth.X_NORMAL, M, K, seed=8)
    assert np.array_equal(run_w4a4(w, X), run_w4a4(w, X))


def test_w4a4_plan_limits():
    d = torch.cuda.current_device()
    bad = [(1, 1024, 512, nv.NVFP4_VARIANT_TC), (1, 1024, 512, nv.NVFP4_VARIANT_GEMV),
           (1, 1024, 512, nv.NVFP4_VARIANT_ROW), (1, 1024, 512, nv.NVFP4_PLAN_WEIGHT_FP8)]
    for M, N, K, flags in bad:
        with pytest.raises(nv.Nvfp4Error) as e:
            nv.nvfp4_linear_plan(M, N, K, d, nv.NVFP4_PLAN_ACT_NVFP4 | flags)
        assert e.value.status == nv.NVFP4_ERR_UNSUPPORTED, (M, N, K, flags)
