"""GPU parity on X rows of wide dynamic range: the hi/lo X planes.

The tensor-core variants take X as f16. Each token row is scaled by a power
of two so that its largest magnitude sits at 2^14; the f16 hi plane holds
that (exact within 2^28 of the maximum) and a lo plane, scaled by 2^29,
holds the remainder (exact down to 2^57 below the maximum). Below that an
element keeps only the lo plane's subnormal step: its absolute error is at
most 2^-68 of the row's largest magnitude, and the header bounds Y there by
the tolerance plus 2^-67 * max_k|x[m][k]| * sum_k|w_hat[n][k]|.

These tests give some tokens a few huge elements (up to 2^40) in columns
where every weight is zero, and small elements (down to 2^-15) everywhere
else: y_ref is then carried by the small elements alone, which only the lo
plane represents, and an output that dropped the lo plane (about 0) fails
the stated tolerance. Every variant and every token class runs: M = 1, 4
(X staged per CTA), M = 5, 8, 16 (X through the ring), K = 5120 (one slice)
and K = 17408 (several K-slices for the staged classes).
"""
import numpy as np
import pytest
import torch

import nvfp4_weight_streaming_b200 as nv
import oracle
import synth
from tests.gpu_util import Weights, check_tolerance, run_linear

pytestmark = pytest.mark.gpu

VARIANTS = [nv.NVFP4_VARIANT_GEMV, nv.NVFP4_VARIANT_MMA, nv.NVFP4_VARIANT_TC, nv.NVFP4_VARIANT_ROW]
VNAME = {0: "auto", 1: "gemv", 2: "mma", 3: "tc", 4: "row"}


def variants_for(M, N, K):
    vs = []
    for v in VARIANTS:
        try:
            p = nv.nvfp4_linear_plan(M, N, K, torch.cuda.current_device(), v)
        except nv.Nvfp4Error as e:
            if e.status == nv.NVFP4_ERR_UNSUPPORTED:
                continue
            raise
        nv.nvfp4_linear_destroy(p)
        vs.append(v)
    return vs + [nv.NVFP4_VARIANT_AUTO]


def wide_x(M, K, wide_tokens, big_cols, seed, small_exp=(-15, -5), big_exp=(10, 40)):
    """bf16 X [M][K]: tokens in `wide_tokens` hold small elements with
    exponents in [small_exp) everywhere and huge ones (the largest exactly
    2^big_exp[1]) at `big_cols`; the other tokens are N(0,1)."""
    rng = np.random.default_rng(seed)
    X = synth.x_bf16_custom(synth.X_NORMAL, M, K, seed=seed)
    for m in wide_tokens:
        mant = rng.uniform(1.0, 2.0, K)
        sign = rng.choice([-1.0, 1.0], K)
        x = sign * mant * np.exp2(rng.integers(small_exp[0], small_exp[1], K).astype(np.float64))
        x[big_cols] = sign[big_cols] * mant[big_cols] * np.exp2(
            rng.integers(big_exp[0], big_exp[1], len(big_cols)).astype(np.float64))
        x[big_cols[0]] = 2.0 ** big_exp[1]
        X[m] = oracle.bf16_round_array(x)
    return X


def weights_zero_at(N, K, cols, seed):
    W = synth.normal_f32(N * K, 0.02, seed=seed, stream=7).reshape(N, K)
    W[:, cols] = 0.0
    return oracle.quantize(W)


CASES = [
    # (M, K, N, tokens with a wide range)
    (1, 5120, 2339, [0]),
    (4, 5120, 2339, [1, 3]),
    (5, 5120, 2339, [0, 4]),
    (8, 5120, 2339, [0, 3, 7]),
    (16, 5120, 2339, [0, 5, 9, 15]),
    (1, 17408, 1024, [0]),
    (4, 17408, 1024, [0, 2]),
    (8, 17408, 1024, [6]),
    (16, 17408, 1024, [1, 14]),
]


@pytest.mark.parametrize("M,K,N,wide", CASES)
def test_lo_plane_carries_small_elements(M, K, N, wide):
    rng = np.random.default_rng(K + M)
    big_cols = np.sort(rng.choice(K, 6, replace=False))
    packed, scales, gs = weights_zero_at(N, K, big_cols, seed=M)
    D = oracle.dequant_f64(packed, scales, gs, N, K)
    assert not D[:, big_cols].any()
    X = wide_x(M, K, wide, big_cols, seed=100 + M)
    y_ref, ad = oracle.linear(packed, scales, gs, X, M, N, K)
    tol = oracle.tolerance(y_ref, ad)
    # the test is sensitive: for the wide tokens a zero output (lo plane
    # dropped) is out of tolerance almost everywhere
    for m in wide:
        assert np.mean(np.abs(y_ref[m]) > tol[m]) > 0.95
    w = Weights(packed, scales, gs)
    for v in variants_for(M, N, K):
        y, ok, _ = run_linear(w, X, v)
        assert ok, VNAME[v]
        check_tolerance(y, y_ref, ad)


@pytest.mark.parametrize("M", [1, 4, 8, 16])
def test_lo_plane_exact_dyadic(M):
    """Small integers times powers of two spread over 2^-16 .. 2^40 in the
    wide tokens, codes 0..15 and scales 1 or 2 with gs = 1: every product
    and every partial sum of the small elements is a dyadic rational exact
    in fp32, and the huge elements meet zero weights, so Y is the oracle's
    value rounded once to bf16 on every variant, bit for bit."""
    N, K = 512, 1024
    codes = np.array([[(3 * n + k) % 16 for k in range(K)] for n in range(N)], np.uint8)
    big_cols = np.array([5, 300, 777])
    codes[:, big_cols] = 0
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    scales = np.array([[0x38 if (n + b) % 3 else 0x40 for b in range(K // 16)] for n in range(N)],
                      np.uint8)
    xs = np.array([[((k * 7 + m) % 9) - 4 for k in range(K)] for m in range(M)], np.float64) * 2.0 ** -12
    wide = list(range(0, M, 2))
    for m in wide:
        xs[m, big_cols] = [2.0 ** 40, -2.0 ** 33, 2.0 ** 20]
    X = oracle.bf16_round_array(xs)
    y_ref, _ = oracle.linear(packed, scales, 1.0, X, M, N, K)
    expect = oracle.bf16_round_array(y_ref)
    assert np.abs(oracle.bf16_bits_to_f64(expect)).max() > 0
    w = Weights(packed, scales, 1.0)
    for v in variants_for(M, N, K):
        y, ok, _ = run_linear(w, X, v)
        assert ok and np.array_equal(y, expect), VNAME[v]


@pytest.mark.parametrize("M", [1, 8, 16])
def test_beyond_two_to_57_meets_the_documented_bound(M):
    """Elements 60..70 binades below their row's maximum (2^40) lie outside
    the exact range of the two planes. The header bounds the error there by
    the stated tolerance plus 2^-67 * max|x_m| * sum_k |w_hat[n][k]| (2^-68
    per element, doubled to cover the final bf16 rounding of that error);
    the GEMV variant (fp32 FMA) meets the plain tolerance."""
    N, K = 768, 5120
    rng = np.random.default_rng(57)
    big_cols = np.sort(rng.choice(K, 4, replace=False))
    packed, scales, gs = weights_zero_at(N, K, big_cols, seed=9)
    wide = [0] if M == 1 else [0, M - 1]
    X = wide_x(M, K, wide, big_cols, seed=300 + M, small_exp=(-30, -20), big_exp=(30, 40))
    y_ref, ad = oracle.linear(packed, scales, gs, X, M, N, K)
    tol = oracle.tolerance(y_ref, ad)
    absw = np.abs(oracle.dequant_f64(packed, scales, gs, N, K)).sum(axis=1)
    xmax = np.abs(oracle.bf16_bits_to_f64(X)).max(axis=1)
    extra = np.outer(xmax, absw) * 2.0 ** -67
    w = Weights(packed, scales, gs)
    for v in variants_for(M, N, K):
        y, ok, _ = run_linear(w, X, v)
        assert ok, VNAME[v]
        yg = oracle.bf16_bits_to_f64(y)
        err = np.abs(yg - y_ref)
        if v == nv.NVFP4_VARIANT_GEMV:
            assert (err <= tol).all()
        assert (err <= tol + extra).all(), VNAME[v]
        narrow = [m for m in range(M) if m not in wide]
        if narrow:
            assert (err[narrow] <= tol[narrow]).all(), VNAME[v]
