"""GPU parity of the fused epilogues against the oracle.

SwiGLU (fused gate+up projection; rows 2c and 2c+1 of W are the gate and up
rows of output column c): every output within swiglu_tolerance of the
oracle's fp64 silu(gate) * up. Argmax (greedy choice over the output rows):
per token the oracle's top row wherever its top-2 gap exceeds the two
logits' bounds, otherwise a row whose exact logit is within those bounds of
the top; the reported value within the logit's bound; exact ties to the
lower row.
"""
import numpy as np
import pytest
import torch

import nvfp4_weight_streaming_b200 as nv
import oracle
import synth
from tests.gpu_util import Guarded, Weights, dev, host_u16

pytestmark = pytest.mark.gpu

_cache = {}


def _weights(name):
    if name not in _cache:
        _cache[name] = oracle.quantize(synth.weights_f32(synth.WORKLOADS[name]))
    return _cache[name]


def _run(w, X, flags, out_count, out_dtype=torch.int16):
    M = X.shape[0]
    plan = nv.nvfp4_linear_plan(M, w.N, w.K, torch.cuda.current_device(), flags)
    try:
        assert nv.nvfp4_linear_variant(plan) == nv.NVFP4_VARIANT_MMA
        wsb = nv.nvfp4_linear_workspace_bytes(plan)
        ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
        y = Guarded(out_count)
        nv.nvfp4_linear_run(plan, w.packed, w.scales, w.gsd, dev(X), y.view, ws, wsb)
        assert nv.nvfp4_linear_status(plan, ws) == nv.NVFP4_OK
        assert y.guards_intact()
        return y.view.clone()
    finally:
        nv.nvfp4_linear_destroy(plan)


def check_swiglu(packed, scales, gs, X, flags=nv.NVFP4_PLAN_EPI_SWIGLU):
    M, K = X.shape
    N = packed.shape[0]
    w = Weights(packed, scales, gs)
    y = _run(w, X, flags, M * (N // 2))
    got = oracle.bf16_bits_to_f64(host_u16(y).reshape(M, N // 2))
    h, g, u, adg, adu = oracle.swiglu_linear(packed, scales, gs, X, M, N, K)
    tol = oracle.swiglu_tolerance(h, g, u, adg, adu)
    bad = ~(np.abs(got - h) <= tol)
    assert not bad.any(), "%d of %d out of tolerance, first %s" % (
        bad.sum(), bad.size, [tuple(i) for i in np.argwhere(bad)[:3]])


@pytest.mark.parametrize("M", [1, 8, 16])
def test_swiglu_decode_projection(M):
    packed, scales, gs = _weights("decode")
    X = synth.x_bf16(synth.WORKLOADS["verify"], M)
    check_swiglu(packed, scales, gs, X)


@pytest.mark.parametrize("M,N,K", [(1, 520, 512), (3, 1000, 768), (5, 130, 256), (16, 778, 1280),
                                   (2, 2, 256), (9, 4098, 512)])
def test_swiglu_ragged_and_split(M, N, K):
    W = synth.normal_f32(N * K, 0.5, seed=17, stream=7).reshape(N, K)
    packed, scales, gs = oracle.quantize(W)
    X = synth.x_bf16_custom(synth.X_OUTLIERS, M, K, seed=19, n_outliers=4, gain=20.0)
    check_swiglu(packed, scales, gs, X)


def test_swiglu_wide_x_uses_the_lo_plane():
    """Tokens spanning 2^40 .. 2^-15 with zero weights at the huge elements:
    the gate and up values come from the lo plane alone."""
    N, K, M = 1024, 5120, 4
    rng = np.random.default_rng(3)
    big = np.sort(rng.choice(K, 5, replace=False))
    W = synth.normal_f32(N * K, 0.5, seed=23, stream=7).reshape(N, K)
    W[:, big] = 0.0
    packed, scales, gs = oracle.quantize(W)
    X = synth.x_bf16_custom(synth.X_NORMAL, M, K, seed=29)
    for m in (0, 3):
        mant = rng.uniform(1.0, 2.0, K)
        x = rng.choice([-1.0, 1.0], K) * mant * np.exp2(rng.integers(-15, -5, K).astype(np.float64))
        x[big] = 2.0 ** 40
        X[m] = oracle.bf16_round_array(x)
    check_swiglu(packed, scales, gs, X)


def check_argmax(packed, scales, gs, X, y_ref=None, absdot=None):
    M, K = X.shape
    N = packed.shape[0]
    w = Weights(packed, scales, gs)
    out = _run(w, X, nv.NVFP4_PLAN_EPI_ARGMAX, 4 * M).cpu().numpy().view(np.uint8)
    idx = out[:4 * M].view(np.int32).copy()
    val = out[4 * M:].view(np.float32).astype(np.float64)
    if y_ref is None:
        y_ref, absdot = oracle.linear(packed, scales, gs, X, M, N, K)
    tol = oracle.tolerance(y_ref, absdot)
    top, decided = oracle.argmax_decided(y_ref, tol)
    for m in range(M):
        j = int(idx[m])
        assert 0 <= j < N
        if decided[m]:
            assert j == top[m], (m, j, int(top[m]))
        else:
            assert y_ref[m, top[m]] - y_ref[m, j] <= tol[m, top[m]] + tol[m, j], (m, j, int(top[m]))
        assert abs(val[m] - y_ref[m, j]) <= tol[m, j], (m, val[m], y_ref[m, j])
    return idx, decided


_lm = {}


def lm_head_weights():
    if "w" not in _lm:
        wl = synth.WORKLOADS["lm_head"]
        ch = 16384
        spans = [slice(r, min(r + ch, wl.N)) for r in range(0, wl.N, ch)]
        gs = max(oracle.global_scale(synth.weights_f32(wl, rows=sp)) for sp in spans)
        packed = np.empty((wl.N, wl.K // 2), np.uint8)
        scales = np.empty((wl.N, wl.K // 16), np.uint8)
        for sp in spans:
            p, s = oracle.quantize_rows(synth.weights_f32(wl, rows=sp), gs)
            packed[sp] = p
            scales[sp] = s
        _lm["w"] = (packed, scales, gs)
    return _lm["w"]


@pytest.mark.parametrize("M", [1, 8, 16])
def test_argmax_lm_head(M):
    """The workload as it is: its 248,320 logits are so close that the top-2
    gap never exceeds the stated bounds, so every token checks the near-tie
    rule; then each token gets one planted row aligned with its X (0.02 *
    sign(x), quantised with the workload's global scale) that leads by far,
    and the GPU must name exactly that row."""
    packed, scales, gs = lm_head_weights()
    wl = synth.WORKLOADS["lm_head"]
    X = synth.x_bf16(wl, M)
    check_argmax(packed, scales, gs, X)
    packed = packed.copy()
    scales = scales.copy()
    xs = oracle.bf16_bits_to_f64(X)
    rows = [1000 + 15013 * m for m in range(M)]
    planted = np.stack([(0.02 * np.sign(xs[m])).astype(np.float32) for m in range(M)])
    p, s = oracle.quantize_rows(planted, gs)
    packed[rows] = p
    scales[rows] = s
    idx, decided = check_argmax(packed, scales, gs, X)
    assert decided.all()
    assert list(idx) == rows


@pytest.mark.parametrize("M,N,K", [(1, 777, 1280), (4, 3000, 512), (16, 4097, 768), (2, 1, 256)])
def test_argmax_ragged_and_split(M, N, K):
    W = synth.normal_f32(N * K, 0.1, seed=31, stream=7).reshape(N, K)
    packed, scales, gs = oracle.quantize(W)
    X = synth.x_bf16_custom(synth.X_RMSNORM, M, K, seed=37)
    check_argmax(packed, scales, gs, X)


def test_argmax_exact_tie_goes_to_the_lower_row():
    """Rows 261 and 266 (one 16-row group) are identical and dominate every
    other row: their sums are bit-identical, and the lower row must win; a
    later call on the same workspace must give the same answer."""
    M, N, K = 3, 1200, 1024
    W = synth.normal_f32(N * K, 0.02, seed=41, stream=7).reshape(N, K)
    W[266] = W[261] = np.abs(W[261]) * 8.0
    packed, scales, gs = oracle.quantize(W)
    assert np.array_equal(packed[261], packed[266]) and np.array_equal(scales[261], scales[266])
    X = np.full((M, K), 0x3F80, np.uint16)                 # x = 1: the all-positive rows lead
    idx, decided = check_argmax(packed, scales, gs, X)
    assert list(idx) == [261] * M
    idx2, _ = check_argmax(packed, scales, gs, X)
    assert list(idx2) == [261] * M


def test_argmax_state_is_cleared_between_calls():
    """One plan and workspace, two calls: the second call's winner has a
    smaller logit than the first call's, so a running maximum left over from
    the first call would be reported again."""
    M, N, K = 2, 2000, 512
    W = synth.normal_f32(N * K, 0.02, seed=43, stream=7).reshape(N, K)
    W[700] = np.abs(W[700]) * 8.0
    packed, scales, gs = oracle.quantize(W)
    w = Weights(packed, scales, gs)
    Xa = np.full((M, K), 0x3F80, np.uint16)                # +1: row 700 leads by far
    Xb = np.full((M, K), 0xBF80, np.uint16)                # -1: row 700 is the smallest
    y_a, ad_a = oracle.linear(packed, scales, gs, Xa, M, N, K)
    y_b, ad_b = oracle.linear(packed, scales, gs, Xb, M, N, K)
    assert y_b.max() < y_a[:, 700].min()
    plan = nv.nvfp4_linear_plan(M, N, K, torch.cuda.current_device(), nv.NVFP4_PLAN_EPI_ARGMAX)
    try:
        wsb = nv.nvfp4_linear_workspace_bytes(plan)
        ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
        outs = []
        for X in (Xa, Xb):
            y = torch.zeros(4 * M, dtype=torch.int16, device="cuda")
            nv.nvfp4_linear_run(plan, w.packed, w.scales, w.gsd, dev(X), y, ws, wsb)
            assert nv.nvfp4_linear_status(plan, ws) == nv.NVFP4_OK
            outs.append(y.cpu().numpy().view(np.uint8)[:4 * M].view(np.int32).copy())
    finally:
        nv.nvfp4_linear_destroy(plan)
    tol_b = oracle.tolerance(y_b, ad_b)
    top_b, dec_b = oracle.argmax_decided(y_b, tol_b)
    assert list(outs[0]) == [700] * M
    for m in range(M):
        assert outs[1][m] != 700
        assert (outs[1][m] == top_b[m]) or not dec_b[m]


def test_epilogue_argument_checks():
    d = torch.cuda.current_device()
    with pytest.raises(nv.Nvfp4Error) as e:
        nv.nvfp4_linear_plan(1, 1001, 256, d, nv.NVFP4_PLAN_EPI_SWIGLU)
    assert e.value.status == nv.NVFP4_ERR_INVALID_ARG
    with pytest.raises(nv.Nvfp4Error) as e:
        nv.nvfp4_linear_plan(1, 1000, 256, d, nv.NVFP4_PLAN_EPI_SWIGLU | nv.NVFP4_PLAN_EPI_ARGMAX)
    assert e.value.status == nv.NVFP4_ERR_INVALID_ARG
    for v in (nv.NVFP4_VARIANT_GEMV, nv.NVFP4_VARIANT_TC, nv.NVFP4_VARIANT_ROW):
        with pytest.raises(nv.Nvfp4Error) as e:
            nv.nvfp4_linear_plan(1, 1000, 256, d, v | nv.NVFP4_PLAN_EPI_ARGMAX)
        assert e.value.status == nv.NVFP4_ERR_UNSUPPORTED


def test_epilogues_with_k_zero():
    d = torch.cuda.current_device()
    dummy = torch.zeros(16, dtype=torch.uint8, device="cuda")
    gsd = torch.ones(1, dtype=torch.float32, device="cuda")
    for flags, count in ((nv.NVFP4_PLAN_EPI_SWIGLU, 2 * 4), (nv.NVFP4_PLAN_EPI_ARGMAX, 4 * 2)):
        plan = nv.nvfp4_linear_plan(2, 8, 0, d, flags)
        try:
            y = Guarded(count)
            nv.nvfp4_linear_run(plan, dummy, dummy, gsd, dummy, y.view)
            torch.cuda.synchronize()
            assert y.guards_intact() and int(y.view.count_nonzero()) == 0
        finally:
            nv.nvfp4_linear_destroy(plan)
