"""nvfp4_linear_run_static: the linear with its split-K scratch in the
library's fixed device array, checked against nvfp4_linear_run with a caller
workspace on the same plan. The reductions are deterministic, so the two
entry points must agree bit for bit, and both must meet the oracle's
tolerance. Two calls in a row must both match (the second one finds the
first one's leftovers in the shared array), also after a run that timed out
and left its counters behind.

Collected last on purpose: it must pass in a fresh process and after every
other test has used the device.
"""
import pytest
import torch

import nvfp4_weight_streaming_b200 as nv
import oracle
import synth
from tests.gpu_util import Guarded, Weights, check_tolerance, dev, host_u16, run_linear

pytestmark = pytest.mark.gpu

CASES = [
    # (variant, M, N, K): split-K plans that use the scratch, and one that needs none
    (nv.NVFP4_VARIANT_MMA, 4, 1024, 8192),
    (nv.NVFP4_VARIANT_MMA, 8, 1024, 8192),      # X planes in the scratch too
    (nv.NVFP4_VARIANT_TC, 16, 1024, 8192),
    (nv.NVFP4_VARIANT_AUTO, 3, 777, 1280),
    (nv.NVFP4_VARIANT_GEMV, 1, 520, 512),
    (nv.NVFP4_VARIANT_ROW, 1, 2339, 5120),      # K-split: row-group counters and partials
    (nv.NVFP4_VARIANT_ROW, 1, 1024, 17408),     # K-split over 17408
]


def _problem(M, N, K, seed):
    W = synth.normal_f32(N * K, 0.02, seed=seed, stream=7).reshape(N, K)
    packed, scales, gs = oracle.quantize(W)
    X = synth.x_bf16_custom(synth.X_OUTLIERS, M, K, seed=seed + 1, n_outliers=4, gain=20.0)
    return Weights(packed, scales, gs), X


@pytest.mark.parametrize("variant,M,N,K", CASES)
def test_static_scratch_matches_workspace_entry(variant, M, N, K):
    w, X = _problem(M, N, K, seed=11 + M)
    y_ref, ad = oracle.linear(w.packed_h, w.scales_h, w.gs, X, M, N, K)
    plan = nv.nvfp4_linear_plan(M, N, K, torch.cuda.current_device(), variant)
    try:
        wsb = nv.nvfp4_linear_workspace_bytes(plan)
        assert wsb <= nv.NVFP4_STATIC_SCRATCH_BYTES
        if variant in (nv.NVFP4_VARIANT_MMA, nv.NVFP4_VARIANT_TC, nv.NVFP4_VARIANT_ROW):
            # counters and partial sums of split tiles (and X planes)
            assert wsb > 256, "case must use the scratch beyond the status word"
        y_ws, ok, _ = run_linear(w, X, plan=plan)
        assert ok
        check_tolerance(y_ws, y_ref, ad)

        xd = dev(X)
        stream = torch.cuda.current_stream()
        status = torch.full((2,), -1, dtype=torch.int32, device="cuda")
        outs = []
        for call in range(2):
            y = Guarded(M * N)
            nv.nvfp4_linear_run_static(plan, w.packed, w.scales, w.gsd, xd, y.view,
                                       status[call:call + 1], stream)
            outs.append(y)
        torch.cuda.synchronize()
        assert status.tolist() == [0, 0], "device wait status %s" % status.tolist()
        for y in outs:
            assert y.guards_intact()
            got = host_u16(y.view).reshape(M, N)
            assert (got == y_ws).all(), "static entry differs from the workspace entry"
            check_tolerance(got, y_ref, ad)
    finally:
        nv.nvfp4_linear_destroy(plan)


@pytest.mark.parametrize("variant", [nv.NVFP4_VARIANT_MMA, nv.NVFP4_VARIANT_ROW])
def test_static_scratch_recovers_after_a_timed_out_run(variant):
    """A test-only plan whose producer never signals runs out its bounded
    device waits and reports a nonzero status through status_out, leaving
    counters behind in the shared array; a normal plan of the same shape
    through the static entry then returns status 0 and the right Y, because
    every static call clears the counters first."""
    M, N, K = 1, 2339, 5120
    w, X = _problem(M, N, K, seed=29)
    y_ref, ad = oracle.linear(w.packed_h, w.scales_h, w.gs, X, M, N, K)
    dev_id = torch.cuda.current_device()
    xd = dev(X)
    status = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    stalled = nv.nvfp4_linear_plan(M, N, K, dev_id, variant | nv.NVFP4_PLAN_TEST_STALL)
    try:
        y = Guarded(M * N)
        nv.nvfp4_linear_run_static(stalled, w.packed, w.scales, w.gsd, xd, y.view, status[0:1])
        torch.cuda.synchronize()
        assert int(status[0].item()) != 0
        assert y.guards_intact()
    finally:
        nv.nvfp4_linear_destroy(stalled)
    plan = nv.nvfp4_linear_plan(M, N, K, dev_id, variant)
    try:
        y = Guarded(M * N)
        nv.nvfp4_linear_run_static(plan, w.packed, w.scales, w.gsd, xd, y.view, status[1:2])
        torch.cuda.synchronize()
        assert int(status[1].item()) == 0
        assert y.guards_intact()
        check_tolerance(host_u16(y.view).reshape(M, N), y_ref, ad)
    finally:
        nv.nvfp4_linear_destroy(plan)


W4A4_TC = nv.NVFP4_PLAN_ACT_NVFP4 | nv.NVFP4_VARIANT_TC


def _w4a4_ref(w, X):
    M, K = X.shape
    xp, xs, gsx = oracle.quantize_x(X)
    return oracle.linear_w4a4(w.packed_h, w.scales_h, w.gs, xp, xs, gsx, M, w.N, K)


@pytest.mark.parametrize("M,N,K", [(16, 1024, 8192), (1, 5120, 17408), (5, 300 * 256, 512)])
def test_static_scratch_w4a4_tensor_cores(M, N, K):
    """W4A4 on the FP4 tensor cores: the X blocks, the X amax and the K-split
    partials in the fixed array; bit-identical to the workspace entry."""
    w, X = _problem(M, N, K, seed=31 + M)
    y_ref, ad = _w4a4_ref(w, X)
    plan = nv.nvfp4_linear_plan(M, N, K, torch.cuda.current_device(), W4A4_TC)
    try:
        assert nv.nvfp4_linear_variant(plan) == nv.NVFP4_VARIANT_TC
        assert nv.nvfp4_linear_workspace_bytes(plan) <= nv.NVFP4_STATIC_SCRATCH_BYTES
        y_ws, ok, _ = run_linear(w, X, plan=plan)
        assert ok
        check_tolerance(y_ws, y_ref, ad)
        xd = dev(X)
        status = torch.full((2,), -1, dtype=torch.int32, device="cuda")
        outs = []
        for call in range(2):
            y = Guarded(M * N)
            nv.nvfp4_linear_run_static(plan, w.packed, w.scales, w.gsd, xd, y.view, status[call:call + 1])
            outs.append(y)
        torch.cuda.synchronize()
        assert status.tolist() == [0, 0]
        for y in outs:
            assert y.guards_intact()
            assert (host_u16(y.view).reshape(M, N) == y_ws).all()
    finally:
        nv.nvfp4_linear_destroy(plan)


def test_static_scratch_w4a4_recovers_after_a_timed_out_run():
    """A stalled W4A4 tensor-core plan leaves its status and possibly counters
    in the shared array; the next static call clears them and is right."""
    M, N, K = 1, 5120, 17408                       # K split: per-tile counters in use
    w, X = _problem(M, N, K, seed=41)
    y_ref, ad = _w4a4_ref(w, X)
    dev_id = torch.cuda.current_device()
    xd = dev(X)
    status = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    stalled = nv.nvfp4_linear_plan(M, N, K, dev_id, W4A4_TC | nv.NVFP4_PLAN_TEST_STALL)
    try:
        y = Guarded(M * N)
        nv.nvfp4_linear_run_static(stalled, w.packed, w.scales, w.gsd, xd, y.view, status[0:1])
        torch.cuda.synchronize()
        assert int(status[0].item()) != 0
        assert y.guards_intact()
    finally:
        nv.nvfp4_linear_destroy(stalled)
    plan = nv.nvfp4_linear_plan(M, N, K, dev_id, W4A4_TC)
    try:
        y = Guarded(M * N)
        nv.nvfp4_linear_run_static(plan, w.packed, w.scales, w.gsd, xd, y.view, status[1:2])
        torch.cuda.synchronize()
        assert int(status[1].item()) == 0
        assert y.guards_intact()
        check_tolerance(host_u16(y.view).reshape(M, N), y_ref, ad)
    finally:
        nv.nvfp4_linear_destroy(plan)


def test_static_scratch_rejects_plans_beyond_its_size():
    """A plan whose workspace exceeds the fixed array is refused with
    WORKSPACE and launches nothing."""
    dev_id = torch.cuda.current_device()
    found = None
    sizes = []
    for v in (nv.NVFP4_VARIANT_TC, nv.NVFP4_VARIANT_MMA):
        for N, K in ((1024, 65536), (2048, 65536), (4096, 65536), (8192, 65536),
                     (16384, 32768), (32768, 16384)):
            try:
                p = nv.nvfp4_linear_plan(16, N, K, dev_id, v)
            except nv.Nvfp4Error:
                continue
            wsb = nv.nvfp4_linear_workspace_bytes(p)
            sizes.append((v, N, K, wsb))
            if wsb > nv.NVFP4_STATIC_SCRATCH_BYTES and found is None:
                found = (p, N, K)
            else:
                nv.nvfp4_linear_destroy(p)
    assert found is not None, "no candidate plan exceeds the array: %s" % sizes
    p, N, K = found
    try:
        d = torch.empty(16, dtype=torch.uint8, device="cuda")
        y = Guarded(16 * N)
        s = nv.nvfp4_linear_run_static(p, d, d, d, d, y.view, None, None, check=False)
        assert s == nv.NVFP4_ERR_WORKSPACE
        torch.cuda.synchronize()
        assert y.guards_intact() and bool((y.view == 0x5A5A).all())
    finally:
        nv.nvfp4_linear_destroy(p)


def test_static_scratch_argument_errors():
    L = nv.lib()
    assert L.nvfp4_linear_run_static(None, None, None, None, None, None, None, None) == \
        nv.NVFP4_ERR_INVALID_ARG
    M, N, K = 4, 1024, 8192
    w, X = _problem(M, N, K, seed=5)
    plan = nv.nvfp4_linear_plan(M, N, K, torch.cuda.current_device(), nv.NVFP4_VARIANT_MMA)
    try:
        y = Guarded(M * N)
        st = torch.zeros(2, dtype=torch.int32, device="cuda")
        odd = st.data_ptr() + 1
        s = nv.nvfp4_linear_run_static(plan, w.packed, w.scales, w.gsd, dev(X), y.view, odd,
                                       None, check=False)
        assert s == nv.NVFP4_ERR_MISALIGNED
        s = nv.nvfp4_linear_run_static(plan, w.packed, w.scales, w.gsd, None, y.view, None,
                                       None, check=False)
        assert s == nv.NVFP4_ERR_INVALID_ARG
    finally:
        nv.nvfp4_linear_destroy(plan)
