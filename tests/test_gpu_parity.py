"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Integer work (unpack/scale decode, quantiser codes) must match bit for bit.
Y must satisfy |y - y_ref| <= 1e-2 |y_ref| + 1e-4 sum_k |w_hat x| per element,
and be exact where the arithmetic is exact (one-hot X, dyadic sums).
Every output buffer carries canary guards that must survive the run.
"""
import numpy as np
import pytest
import torch

import nvfp4_weight_streaming_b200 as nv
import oracle
import synth
from tests.gpu_util import Guarded, Weights, check_tolerance, dev, host_u16, run_linear

pytestmark = pytest.mark.gpu

VARIANTS = [nv.NVFP4_VARIANT_GEMV, nv.NVFP4_VARIANT_MMA, nv.NVFP4_VARIANT_TC, nv.NVFP4_VARIANT_ROW]
VNAME = {0: "auto", 1: "gemv", 2: "mma", 3: "tc", 4: "row"}

_cache = {}


def quantized(name: str, copy: int = 0):
    """(packed, scales, gs) of a workload's weights, quantised by the oracle."""
    key = (name, copy)
    if key not in _cache:
        wl = synth.WORKLOADS[name]
        _cache[key] = oracle.quantize(synth.weights_f32(wl, copy))
    return _cache[key]


def supported(variant: int, M: int, N: int, K: int) -> bool:
    try:
        p = nv.nvfp4_linear_plan(M, N, K, torch.cuda.current_device(), variant)
    except nv.Nvfp4Error as e:
        if e.status == nv.NVFP4_ERR_UNSUPPORTED:
            return False
        raise
    nv.nvfp4_linear_destroy(p)
    return True


def variants_for(M, N, K):
    vs = [v for v in VARIANTS if supported(v, M, N, K)]
    assert vs, "no variant supports M=%d N=%d K=%d" % (M, N, K)
    return vs + [nv.NVFP4_VARIANT_AUTO]


# ----- unpack / scale decode (bit exact) -----------------------------------

def pack_check(packed, scales, gs, N, K, with_out=True):
    out = Guarded(N * K) if with_out else None
    bad = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_pack_check(dev(packed), dev(scales),
                        torch.tensor([gs], dtype=torch.float32, device="cuda"), N, K,
                        None if out is None else out.view, bad)
    torch.cuda.synchronize()
    res = None if out is None else host_u16(out.view).reshape(N, K)
    return res, int(bad.item()), (out is None or out.guards_intact())


def test_pack_check_exhaustive_codes_times_scales():
    finite = [c for c in range(256) if c not in (0x7F, 0xFF)]
    N, K = len(finite), 32
    packed = np.zeros((N, K // 2), np.uint8)
    for j in range(K // 2):
        packed[:, j] = ((2 * j) % 16) | (((2 * j + 1) % 16) << 4)
    scales = np.repeat(np.array(finite, np.uint8).reshape(N, 1), 2, axis=1)
    got, bad, ok = pack_check(packed, scales, 1.0, N, K)
    assert ok and bad == 0
    ref = oracle.dequant_bf16_nogs(packed, scales, N, K)
    assert np.array_equal(got, ref)


def test_pack_check_counts_nan_scales_and_bad_global():
    packed = np.random.default_rng(0).integers(0, 256, size=(4, 32), dtype=np.uint8)
    scales = np.array([[0x38, 0x7F, 0x40, 0x38], [0xFF, 0x00, 0x7F, 0x01],
                       [0x38, 0x38, 0x38, 0x38], [0x80, 0xFE, 0x7E, 0x7F]], np.uint8)
    for gs in (1.0, -1.0, float("nan"), float("inf"), 0.0):
        _, bad, _ = pack_check(packed, scales, gs, 4, 64, with_out=False)
        assert bad == oracle.count_bad(scales, gs)
    got, _, ok = pack_check(packed, scales, 1.0, 4, 64)
    ref = oracle.dequant_bf16_nogs(packed, scales, 4, 64)
    finite = np.repeat(~np.isin(scales, [0x7F, 0xFF]), 16, axis=1)
    assert ok and np.array_equal(got[finite], ref[finite])


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_pack_check_workload_weights(name):
    packed, scales, gs = quantized(name)
    N, K = packed.shape[0], packed.shape[1] * 2
    got, bad, ok = pack_check(packed, scales, gs, N, K)
    assert ok and bad == 0
    assert np.array_equal(got, oracle.dequant_bf16_nogs(packed, scales, N, K))


# ----- GPU quantiser (bit exact against the oracle's quantiser) ------------

def gpu_quantize(W):
    N, K = W.shape
    wd = torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda()
    p = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    s = torch.zeros((N, K // 16), dtype=torch.uint8, device="cuda")
    g = torch.zeros(1, dtype=torch.float32, device="cuda")
    bad = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_quantize(wd, N, K, p, s, g, bad)
    torch.cuda.synchronize()
    return p.cpu().numpy(), s.cpu().numpy(), float(g.item()), int(bad.item())


def quantizer_cases():
    rng = np.random.default_rng(11)
    yield "tiny", synth.weights_f32(synth.WORKLOADS["tiny"])
    # magnitudes spread over many binades, so scales hit subnormal and saturated codes
    W = (np.exp2(rng.uniform(-30, 6, (64, 512))) * rng.choice([-1, 1], (64, 512))).astype(np.float32)
    yield "logspread", W
    W = rng.normal(0, 1, (32, 256)).astype(np.float32)
    W[3, 16:32] = 0.0
    W[5, :] = 0.0
    W[7, 40] = -1e-30
    yield "zeros", W
    # exact E2M1 midpoints under a power-of-two scale
    unit = 2.0 ** -8 * 2.0
    mids = np.array([6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75,
                     -2.5, -3.5, -5.0, 0.0])
    W = np.zeros((2, 32), np.float32)
    W[0, :16] = mids * unit
    W[0, 16] = 6.0 * 448.0 * 2.0 ** -8
    W[1, :16] = -mids * unit
    yield "ties", W


@pytest.mark.parametrize("case", list(range(4)))
def test_quantizer_bit_exact(case):
    name, W = list(quantizer_cases())[case]
    p, s, g, bad = gpu_quantize(W)
    rp, rs, rg = oracle.quantize(W)
    assert bad == 0
    assert g == rg, name
    assert np.array_equal(s, rs), name
    assert np.array_equal(p, rp), name


def test_quantizer_bit_exact_decode_weights():
    W = synth.weights_f32(synth.WORKLOADS["decode"])
    p, s, g, bad = gpu_quantize(W)
    rp, rs, rg = quantized("decode")
    assert bad == 0 and g == rg
    assert np.array_equal(s, rs)
    assert np.array_equal(p, rp)


def test_quantizer_flags_nonfinite():
    W = np.zeros((2, 32), np.float32)
    W[0, 3] = np.nan
    W[1, 5] = np.inf
    _, _, _, bad = gpu_quantize(W)
    assert bad == 2


# ----- the linear ----------------------------------------------------------

def tiny_weights():
    return Weights(*quantized("tiny"))


@pytest.mark.parametrize("M", [1, 2, 3, 4, 8, 12, 16])
def test_linear_tiny_all_variants(M):
    w = tiny_weights()
    X = synth.x_bf16_custom(synth.X_NORMAL, M, w.K, seed=M)
    y_ref, ad = oracle.linear(w.packed_h, w.scales_h, w.gs, X, M, w.N, w.K)
    for v in variants_for(M, w.N, w.K):
        y, ok, info = run_linear(w, X, v)
        assert ok, ("guard bytes overwritten", VNAME[v])
        check_tolerance(y, y_ref, ad)


@pytest.mark.parametrize("M,N,K", [(1, 520, 512), (3, 1000, 768), (5, 129, 256), (16, 777, 1280),
                                   (2, 1, 256), (9, 4097, 512),
                                   # 130 and 128 tiles of 256 rows: one whole tile per CTA
                                   (1, 130 * 256 - 77, 512), (2, 130 * 256 - 77, 512),
                                   (16, 127 * 256 + 5, 256)])
def test_linear_ragged_shapes(M, N, K):
    """N not a multiple of any tile; several tiles plus a ragged tail."""
    W = synth.normal_f32(N * K, 0.02, seed=3, stream=7).reshape(N, K)
    packed, scales, gs = oracle.quantize(W)
    w = Weights(packed, scales, gs)
    X = synth.x_bf16_custom(synth.X_OUTLIERS, M, K, seed=5, n_outliers=4, gain=20.0)
    y_ref, ad = oracle.linear(packed, scales, gs, X, M, N, K)
    for v in variants_for(M, N, K):
        y, ok, _ = run_linear(w, X, v)
        assert ok, VNAME[v]
        check_tolerance(y, y_ref, ad)


def test_linear_one_hot_is_exact():
    """X = e_k with gs a power of two: Y[:, n] = bf16(gs * w_hat[n][k]) exactly,
    whatever the summation order."""
    w0 = quantized("tiny")
    w = Weights(w0[0], w0[1], 2.0 ** -12)
    D = oracle.dequant_f64(w.packed_h, w.scales_h, w.gs, w.N, w.K)
    for k in (0, 1, 31, 200, 255):
        X = np.zeros((1, w.K), np.uint16)
        X[0, k] = 0x3F80
        expect = oracle.bf16_round_array(D[:, k])
        for v in variants_for(1, w.N, w.K):
            y, ok, _ = run_linear(w, X, v)
            assert ok and np.array_equal(y[0], expect), (k, VNAME[v])


def test_linear_dyadic_small_integers_exact():
    """Small-integer X, codes cycling through all 16 values, scales 1 or 2,
    gs = 1: every partial sum is an integer or half-integer well inside fp32's
    exact range, so Y equals the oracle's fp64 value rounded once to bf16."""
    M, N, K = 4, 32, 256
    codes = np.array([[(n + k) % 16 for k in range(K)] for n in range(N)], np.uint8)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    scales = np.array([[0x38 if (n + b) % 2 == 0 else 0x40 for b in range(K // 16)]
                       for n in range(N)], np.uint8)
    xs = np.array([[(k % 5) - m for k in range(K)] for m in range(M)], np.float64)
    X = oracle.bf16_round_array(xs)
    y_ref, _ = oracle.linear(packed, scales, 1.0, X, M, N, K)
    expect = oracle.bf16_round_array(y_ref)
    w = Weights(packed, scales, 1.0)
    for v in variants_for(M, N, K):
        y, ok, _ = run_linear(w, X, v)
        assert ok and np.array_equal(y, expect), VNAME[v]


def test_linear_doubling_x_doubles_y_exactly():
    w = tiny_weights()
    X = synth.x_bf16_custom(synth.X_NORMAL, 2, w.K, seed=9)
    X2 = (X.astype(np.uint32) + 0x80).astype(np.uint16)
    X2[(X & 0x7FFF) == 0] = X[(X & 0x7FFF) == 0]
    for v in variants_for(2, w.N, w.K):
        y1, _, _ = run_linear(w, X, v)
        y2, _, _ = run_linear(w, X2, v)
        a = oracle.bf16_bits_to_f64(y1)
        b = oracle.bf16_bits_to_f64(y2)
        assert np.array_equal(2 * a, b), VNAME[v]


@pytest.mark.parametrize("M", [1, 8, 16])
def test_linear_deterministic_and_rows_independent(M):
    """Back-to-back calls on one workspace give bit-identical Y (also catches
    a ring slot refilled while its data is still being read)."""
    packed, scales, gs = quantized("decode")
    w = Weights(packed, scales, gs)
    X = synth.x_bf16(synth.WORKLOADS["verify"], M)
    for v in variants_for(M, w.N, w.K):
        y1, _, _ = run_linear(w, X, v)
        y2, _, _ = run_linear(w, X, v, repeat=3)
        assert np.array_equal(y1, y2), VNAME[v]


@pytest.mark.parametrize("variant,M", [(nv.NVFP4_VARIANT_MMA, 1), (nv.NVFP4_VARIANT_MMA, 4),
                                       (nv.NVFP4_VARIANT_MMA, 16), (nv.NVFP4_VARIANT_ROW, 1),
                                       (nv.NVFP4_VARIANT_ROW, 2)])
def test_pdl_chained_calls_read_the_previous_output(variant, M):
    """Programmatic dependent launch: each call's X is the previous call's Y,
    launched back to back on one stream with one shared workspace. Every
    output must match the oracle applied to the GPU's own previous output, so
    a call that read X, or reused the workspace, before the previous call had
    finished would be caught."""
    K = N = 2048
    chain = 6
    ws_h = []
    for i in range(chain):
        W = synth.normal_f32(N * K, 1.0 / np.sqrt(K), seed=40 + i, stream=7).reshape(N, K)
        ws_h.append(oracle.quantize(W))
    dev_w = [Weights(*q) for q in ws_h]
    X0 = synth.x_bf16_custom(synth.X_NORMAL, M, K, seed=9)
    flags = variant | nv.NVFP4_PLAN_PDL
    plan = nv.nvfp4_linear_plan(M, N, K, torch.cuda.current_device(), flags)
    try:
        wsb = nv.nvfp4_linear_workspace_bytes(plan)
        ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
        bufs = [dev(X0)] + [torch.empty((M, N), dtype=torch.int16, device="cuda") for _ in range(chain)]
        stream = torch.cuda.current_stream()
        for rep in range(3):
            for i in range(chain):
                nv.nvfp4_linear_run(plan, dev_w[i].packed, dev_w[i].scales, dev_w[i].gsd, bufs[i],
                                    bufs[i + 1], ws, wsb, stream)
            assert nv.nvfp4_linear_status(plan, ws, stream) == nv.NVFP4_OK
            for i in range(chain):
                xin = host_u16(bufs[i]).reshape(M, K)
                y_ref, ad = oracle.linear(ws_h[i][0], ws_h[i][1], ws_h[i][2], xin, M, N, K)
                check_tolerance(host_u16(bufs[i + 1]).reshape(M, N), y_ref, ad)
            for b in bufs[1:]:
                b.fill_(0x5A5A)
    finally:
        nv.nvfp4_linear_destroy(plan)


def test_rows_of_y_depend_only_on_their_row_of_x():
    """Row m of Y from an M=16 call against the M=1 call on row m alone: within
    tolerance of each other's oracle values (required); how many rows are bit
    identical is reported, not required (the token classes differ)."""
    packed, scales, gs = quantized("decode")
    w = Weights(packed, scales, gs)
    X = synth.x_bf16(synth.WORKLOADS["verify"], 16)
    rows = np.arange(0, w.N, 97)
    y_ref, ad = oracle.linear(packed, scales, gs, X, 16, w.N, w.K, rows=rows)
    y16, _, _ = run_linear(w, X)
    same = 0
    for m in (0, 5, 15):
        y1, _, _ = run_linear(w, X[m:m + 1])
        check_tolerance(y1[:, rows], y_ref[m:m + 1], ad[m:m + 1])
        check_tolerance(y16[m:m + 1, rows], y_ref[m:m + 1], ad[m:m + 1])
        same += int(np.array_equal(y1[0], y16[m]))
    print("rows bit-identical between M=1 and M=16 calls: %d of 3" % same)


def test_linear_k_zero_writes_zeros_and_n_zero_is_noop():
    w = Weights(np.zeros((8, 0), np.uint8), np.zeros((8, 0), np.uint8), 1.0)
    w.packed = torch.zeros(16, dtype=torch.uint8, device="cuda")
    w.scales = torch.zeros(16, dtype=torch.uint8, device="cuda")
    X = np.zeros((2, 0), np.uint16)
    plan = nv.nvfp4_linear_plan(2, 8, 0, torch.cuda.current_device(), 0)
    try:
        y = Guarded(16)
        xd = torch.zeros(8, dtype=torch.int16, device="cuda")
        nv.nvfp4_linear_run(plan, w.packed, w.scales, w.gsd, xd, y.view)
        torch.cuda.synchronize()
        assert y.guards_intact() and int((y.view != 0).sum()) == 0
    finally:
        nv.nvfp4_linear_destroy(plan)
    plan = nv.nvfp4_linear_plan(1, 0, 256, torch.cuda.current_device(), 0)
    nv.nvfp4_linear_run(plan, None, None, w.gsd, None, w.gsd)
    nv.nvfp4_linear_destroy(plan)


def test_launches_per_run_counts_the_x_conversion_kernel():
    """The mma variant with M >= 5 converts X in a kernel of its own before
    the main kernel; every other plan launches one kernel, N == 0 none."""
    d = torch.cuda.current_device()
    cases = [(nv.NVFP4_VARIANT_MMA, 1, 1024, 5120, 1), (nv.NVFP4_VARIANT_MMA, 4, 1024, 5120, 1),
             (nv.NVFP4_VARIANT_MMA, 5, 1024, 5120, 2), (nv.NVFP4_VARIANT_MMA, 16, 1024, 5120, 2),
             (nv.NVFP4_VARIANT_TC, 16, 1024, 5120, 1), (nv.NVFP4_VARIANT_GEMV, 1, 1024, 5120, 1),
             (nv.NVFP4_VARIANT_MMA, 8, 1024, 0, 1), (nv.NVFP4_VARIANT_AUTO, 1, 0, 256, 0),
             (nv.NVFP4_VARIANT_ROW, 1, 1024, 5120, 1), (nv.NVFP4_VARIANT_ROW, 2, 1024, 5120, 1)]
    for variant, M, N, K, want in cases:
        plan = nv.nvfp4_linear_plan(M, N, K, d, variant)
        try:
            assert nv.nvfp4_linear_launches_per_run(plan) == want, (variant, M, N, K)
        finally:
            nv.nvfp4_linear_destroy(plan)


@pytest.mark.parametrize("variant", [nv.NVFP4_VARIANT_TC, nv.NVFP4_VARIANT_MMA, nv.NVFP4_VARIANT_ROW])
def test_forced_timeout_reports_status_and_recovers(variant):
    """Test-only flag: the TMA producer never signals, every bounded wait runs
    out, the kernel reports NVFP4_ERR_TIMEOUT through the status word and
    returns; the same workspace then serves a normal run."""
    w = tiny_weights()
    X = synth.x_bf16(synth.WORKLOADS["tiny"], 1)
    dev_id = torch.cuda.current_device()
    plan = nv.nvfp4_linear_plan(1, w.N, w.K, dev_id, variant | nv.NVFP4_PLAN_TEST_STALL)
    try:
        wsb = nv.nvfp4_linear_workspace_bytes(plan)
        ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
        y = Guarded(w.N)
        nv.nvfp4_linear_run(plan, w.packed, w.scales, w.gsd, dev(X), y.view, ws, wsb)
        assert nv.nvfp4_linear_status(plan, ws) == nv.NVFP4_ERR_TIMEOUT
        assert y.guards_intact()
        assert int(ws.sum()) == 0                    # cleared by the status call
    finally:
        nv.nvfp4_linear_destroy(plan)
    y_ref, ad = oracle.linear(w.packed_h, w.scales_h, w.gs, X, 1, w.N, w.K)
    got, ok, _ = run_linear(w, X, variant)
    assert ok
    check_tolerance(got, y_ref, ad)


def test_linear_argument_errors_launch_nothing():
    w = tiny_weights()
    plan = nv.nvfp4_linear_plan(1, w.N, w.K, torch.cuda.current_device(), 0)
    try:
        xd = dev(synth.x_bf16(synth.WORKLOADS["tiny"], 1))
        y = Guarded(w.N)
        base = w.packed.data_ptr()
        cases = [
            ((base + 8, w.scales, w.gsd, xd, y.view), nv.NVFP4_ERR_MISALIGNED),
            ((w.packed, w.scales, w.gsd, xd.data_ptr() + 2, y.view), nv.NVFP4_ERR_MISALIGNED),
            ((w.packed, None, w.gsd, xd, y.view), nv.NVFP4_ERR_INVALID_ARG),
            ((w.packed, w.scales, None, xd, y.view), nv.NVFP4_ERR_INVALID_ARG),
            ((w.packed, w.scales, w.gsd, xd, None), nv.NVFP4_ERR_INVALID_ARG),
        ]
        for args, status in cases:
            s = nv.nvfp4_linear_run(plan, *args, check=False)
            assert s == status
        torch.cuda.synchronize()
        assert int((y.view != 0x5A5A).sum()) == 0      # nothing was written
    finally:
        nv.nvfp4_linear_destroy(plan)
    with pytest.raises(nv.Nvfp4Error):
        nv.nvfp4_linear_plan(1, 8, 256, torch.cuda.device_count(), 0)


# ----- full-size workloads ------------------------------------------------

def full_check(name, M, copy=0, rows=None):
    packed, scales, gs = quantized(name, copy)
    w = Weights(packed, scales, gs)
    wl = synth.WORKLOADS[name]
    X = synth.x_bf16(wl, M)
    results = {}
    for v in variants_for(M, w.N, w.K):
        y, ok, info = run_linear(w, X, v)
        assert ok, VNAME[v]
        results[v] = y
    if rows is None:
        y_ref, ad = oracle.linear(packed, scales, gs, X, M, w.N, w.K)
        for v, y in results.items():
            check_tolerance(y, y_ref, ad)
    else:
        y_ref, ad = oracle.linear(packed, scales, gs, X, M, w.N, w.K, rows=rows)
        for v, y in results.items():
            check_tolerance(y[:, rows], y_ref, ad)
    return results


def test_decode_projection_full():
    full_check("decode", 1)


@pytest.mark.parametrize("M", [2, 4, 8, 12, 16])
def test_verify_projection_full(M):
    full_check("verify", M)


@pytest.mark.parametrize("M", [1, 4, 8, 16])
def test_down_projection_full(M):
    full_check("down", M)


# ----- lm_head: N = 248,320 (1.27e9 weights) ------------------------------

_lm = {}


def lm_head_weights():
    """The lm_head workload quantised by the oracle in row chunks (the fp32
    matrix would take 5 GB): the global scale is the largest chunk scale
    (amax / (6 * 448) is monotonic in amax), then each chunk is quantised
    with it."""
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
def test_lm_head_full_logits_and_argmax(M):
    """Every logit within tolerance of the oracle, and per token the argmax
    over all 248,320 logits: the GPU's index is the oracle's, or (a bf16 tie
    or near-tie at the top) one whose exact logit is within tolerance of the
    oracle's maximum."""
    packed, scales, gs = lm_head_weights()
    wl = synth.WORKLOADS["lm_head"]
    if "dev" not in _lm:
        _lm["dev"] = Weights(packed, scales, gs)
    w = _lm["dev"]
    X = synth.x_bf16(wl, M)
    y_ref, ad = oracle.linear(packed, scales, gs, X, M, wl.N, wl.K)
    tol = oracle.tolerance(y_ref, ad)
    for v in variants_for(M, wl.N, wl.K):
        y, ok, _ = run_linear(w, X, v)
        assert ok, VNAME[v]
        check_tolerance(y, y_ref, ad)
        yg = oracle.bf16_bits_to_f64(y)
        for m in range(M):
            jg, jr = int(np.argmax(yg[m])), int(np.argmax(y_ref[m]))
            assert jg == jr or y_ref[m, jr] - y_ref[m, jg] <= tol[m, jr] + tol[m, jg], \
                (VNAME[v], m, jg, jr)
