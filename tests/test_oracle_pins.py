"""Pins for the CPU oracle, each checked against something other than the oracle.

Sources of truth used here:
  * the E2M1 grid of the OCP Microscaling spec (tests/golden/e2m1_grid.txt);
  * PyTorch's float8_e4m3fn and bfloat16 conversions (independent library code);
  * brute-force searches written in this file;
  * closed forms (on-grid round trips, one-hot inputs, dyadic sums);
  * the sizes printed on page "Qwen3.8-27B-NVFP4-RTX5090 API & Inference
    Endpoint", section "Why lm_head is NVFP4, and why MTP is gone".
Nothing here calls back into the function under test to produce its expectation.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.conftest import read_golden



def grid():
    rows = read_golden("e2m1_grid.txt")
    return {int(c): float(v) for c, v in rows}


def torch_e4m3_value(code):
    t = torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn)
    return float(t.to(torch.float64)[0])


def torch_bf16_bits(v):
    t = torch.tensor([v], dtype=torch.float64).to(torch.bfloat16)
    return int(t.view(torch.int16)[0]) & 0xFFFF


# ----- decode -------------------------------------------------------------

def test_e2m1_decode_matches_ocp_grid():
    g = grid()
    for code in range(16):
        v = oracle.e2m1_decode(code)
        assert v == g[code]
        assert math.copysign(1.0, v) == math.copysign(1.0, g[code])   # -0.0 for 0x8


def test_e4m3_decode_matches_torch_all_codes():
    for code in range(256):
        ref = torch_e4m3_value(code)
        v = oracle.e4m3_decode(code)
        if math.isnan(ref):
            assert math.isnan(v) and oracle.e4m3_is_nan(code)
            assert code in (0x7F, 0xFF)
        else:
            assert v == ref, hex(code)
            assert not oracle.e4m3_is_nan(code)
    assert oracle.e4m3_decode(0x7E) == 448.0            # largest finite
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9        # smallest subnormal


def test_dequant_bf16_products_exhaustive():
    """All 16 nibble codes x all 254 finite E4M3 codes: the bf16 product equals
    the exact product (torch decode, torch rounding) and is exact in bf16."""
    g = grid()
    finite = [c for c in range(256) if c not in (0x7F, 0xFF)]
    N = len(finite)
    K = 16
    # row i: scale = finite[i]; the 16 elements are codes 0..15 in order.
    packed = np.zeros((N, K // 2), np.uint8)
    for j in range(K // 2):
        packed[:, j] = (2 * j) | ((2 * j + 1) << 4)
    scales = np.array(finite, np.uint8).reshape(N, 1)
    out = oracle.dequant_bf16_nogs(packed, scales, N, K)
    for i, sc in enumerate(finite):
        s = torch_e4m3_value(sc)
        for code in range(16):
            exact = g[code] * s
            bits = torch_bf16_bits(exact)
            assert int(out[i, code]) == bits, (hex(sc), code)
            back = float(np.array([bits << 16], np.uint32).view(np.float32)[0])
            assert back == exact            # the product is representable in bf16


# ----- encode -------------------------------------------------------------

def brute_e2m1(r):
    """Argmin over the 16 codes of |r - value|, ties to the even code, saturating."""
    g = grid()
    if r >= 6.0:
        return 7
    if r <= -6.0:
        return 15
    best = None
    for code in range(16):
        d = abs(float(np.float64(r)) - g[code])
        key = (d, code % 2)
        if best is None or key < best[0]:
            best = (key, code)
    code = best[1]
    if g[code] == 0.0:
        return 0
    # prefer the code whose sign matches r among equal values
    return code


def test_e2m1_encode_ties_golden():
    g = grid()
    for r, v in read_golden("e2m1_ties.txt"):
        code = oracle.e2m1_encode(float(r))
        assert g[code] == float(v), r
    assert oracle.e2m1_encode(-0.1) == 0          # negative results round to +0 code
    assert oracle.e2m1_encode(-0.0) == 0


def test_e2m1_encode_bruteforce_random():
    rng = np.random.default_rng(1)
    vals = np.concatenate([rng.uniform(-8, 8, 20000), rng.normal(0, 2, 5000),
                           np.array([0.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0])])
    vals = vals.astype(np.float32)
    g = grid()
    for r in vals:
        code = oracle.e2m1_encode(float(r))
        ref = brute_e2m1(float(r))
        assert g[code] == g[ref] or (g[code] == 0 and g[ref] == 0), r
        if g[code] != 0:
            assert (code >= 8) == (r < 0)


def brute_e4m3(u):
    """Nearest finite E4M3 value (decoded by torch), ties to the even code, saturating."""
    a = abs(float(u))
    if a >= 448.0:
        mag = 0x7E
    else:
        best = None
        for c in range(0x7F):
            d = abs(a - torch_e4m3_value(c))
            key = (d, c % 2)
            if best is None or key < best[0]:
                best = (key, c)
        mag = best[1]
    return (0x80 if math.copysign(1.0, u) < 0 else 0) | mag


def test_e4m3_encode_bruteforce():
    rng = np.random.default_rng(2)
    vals = list(np.exp2(rng.uniform(-12, 9.5, 3000)).astype(np.float32))
    # every midpoint between adjacent finite magnitudes, and the values themselves
    mags = [torch_e4m3_value(c) for c in range(0x7F)]
    for lo, hi in zip(mags[:-1], mags[1:]):
        vals.append(np.float32((lo + hi) / 2))
        vals.append(np.float32(lo))
    vals += [np.float32(448.0), np.float32(460.0), np.float32(1e9), np.float32(0.0)]
    for u in vals:
        assert oracle.e4m3_encode(float(u)) == brute_e4m3(float(u)), float(u)


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(3)
    u = np.exp2(rng.uniform(-11, 8.7, 5000)).astype(np.float32)
    u = u[u < 448.0]
    ref = torch.from_numpy(u).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(t)) for t in u], np.uint8)
    assert np.array_equal(got, ref)


def test_bf16_rne_matches_torch():
    rng = np.random.default_rng(4)
    f = np.concatenate([rng.normal(0, 1, 4000), np.exp2(rng.uniform(-140, 127, 4000)) *
                        rng.choice([-1, 1], 4000)]).astype(np.float32)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([oracle.bf16_rne(float(t)) for t in f], np.uint16)
    assert np.array_equal(got, ref)
    assert oracle.bf16_rne(3.5e38) == 0x7F80
    assert oracle.bf16_rne(-0.0) == 0x8000


# ----- quantiser ----------------------------------------------------------

def on_grid_tensor(N=8, K=64, gs=2.0 ** -10, seed=5):
    """W whose every element is e2m1 * e4m3 * gs exactly; every block holds a
    +-6 code, and block (0,0) has scale 448 so amax(W) = 6*448*gs."""
    rng = np.random.default_rng(seed)
    g = grid()
    codes = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    codes[:, ::16] = np.where(rng.integers(0, 2, size=(N, K // 16)) == 1, 7, 15)
    finite_pos = [c for c in range(1, 0x7F)]
    scodes = rng.choice(finite_pos, size=(N, K // 16)).astype(np.uint8)
    scodes[0, 0] = 0x7E
    vals = np.vectorize(lambda c: g[int(c)])(codes)
    svals = np.vectorize(torch_e4m3_value)(scodes)
    W = (vals * np.repeat(svals, 16, axis=1) * gs).astype(np.float32)
    assert np.all(W.astype(np.float64) == vals * np.repeat(svals, 16, axis=1) * gs)
    codes = np.where(vals == 0.0, 0, codes).astype(np.uint8)   # -0 codes become 0
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return W, packed, scodes, gs


def test_quantize_round_trip_on_grid():
    W, packed, scodes, gs = on_grid_tensor()
    p, s, g = oracle.quantize(W)
    assert g == gs
    assert np.array_equal(s, scodes)
    assert np.array_equal(p, packed)


def test_quantize_zero_block_and_zero_tensor():
    W, _, _, _ = on_grid_tensor()
    W[3, 16:32] = 0.0
    p, s, g = oracle.quantize(W)
    assert s[3, 1] == 0
    assert np.all(p[3, 8:16] == 0)
    z = np.zeros((4, 32), np.float32)
    p, s, g = oracle.quantize(z)
    assert g == 0.0 and not p.any() and not s.any()


def test_quantize_rejects_nonfinite():
    w = np.zeros((2, 16), np.float32)
    w[1, 3] = np.inf
    with pytest.raises(ValueError):
        oracle.quantize(w)


def test_quantize_tie_codes():
    """Block with amax = 6*s*gs and elements on exact E2M1 midpoints."""
    gs = 2.0 ** -8
    s = 2.0                                      # E4M3 code 0x40
    unit = s * gs
    mids = [6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75,
            -2.5, -3.5, -5.0, 0.0]
    w = np.zeros((1, 32), np.float32)
    w[0, :16] = np.array(mids) * unit
    w[0, 16] = 6.0 * 448.0 * gs                  # sets amax so that gs comes out exact
    p, sc, g = oracle.quantize(w)
    assert g == gs and sc[0, 0] == 0x40
    gr = grid()
    codes = [(p[0, j // 2] >> (4 * (j % 2))) & 0xF for j in range(16)]
    expect = [6.0, 0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 0.0, -1.0, -1.0, -2.0, -2.0, -4.0,
              -4.0, 0.0]
    assert [gr[int(c)] for c in codes] == expect
    assert codes[1] == 0 and codes[8] == 0       # no negative-zero codes


def test_quantize_scale_choice_bruteforce():
    """For random blocks the chosen scale code is the E4M3 nearest (ties even) to
    the fp32 value (amax_b / 6) / gs, found by brute force."""
    wl = synth.WORKLOADS["tiny"]
    W = synth.weights_f32(wl)
    p, s, gs = oracle.quantize(W)
    assert gs == np.float32(np.abs(W).max()) / np.float32(2688.0)
    amax_b = np.abs(W.reshape(wl.N, wl.K // 16, 16)).max(axis=2)
    for n in range(0, wl.N, 37):
        for b in range(wl.K // 16):
            u = np.float32(np.float32(amax_b[n, b]) / np.float32(6.0)) / np.float32(gs)
            assert s[n, b] == brute_e4m3(float(np.float32(u)))


def test_quantize_codes_are_nearest_to_decoded_scale():
    """Every code is the E2M1 nearest of w / (dec(s) * gs) (fp32), by brute force."""
    wl = synth.WORKLOADS["tiny"]
    W = synth.weights_f32(wl)[:40]
    p, s, gs = oracle.quantize(W)
    for n in range(W.shape[0]):
        for k in range(0, W.shape[1], 3):
            denom = np.float32(np.float32(torch_e4m3_value(int(s[n, k // 16]))) * np.float32(gs))
            r = np.float32(W[n, k]) / denom
            code = (p[n, k // 2] >> (4 * (k % 2))) & 0xF
            assert grid()[int(code)] == grid()[brute_e2m1(float(r))]


# ----- dequant and linear -------------------------------------------------

def independent_dequant(packed, scales, gs, N, K):
    g = grid()
    lo = packed & 0xF
    hi = packed >> 4
    codes = np.empty((N, K), np.uint8)
    codes[:, 0::2] = lo
    codes[:, 1::2] = hi
    vals = np.vectorize(lambda c: g[int(c)])(codes)
    svals = np.vectorize(torch_e4m3_value)(scales)
    return vals * np.repeat(svals, 16, axis=1) * np.float64(gs)


def test_dequant_matches_independent_decode():
    wl = synth.WORKLOADS["tiny"]
    p, s, gs = oracle.quantize(synth.weights_f32(wl))
    ref = independent_dequant(p, s, gs, wl.N, wl.K)
    got = oracle.dequant_f64(p, s, gs, wl.N, wl.K)
    assert np.array_equal(got, ref)


def test_linear_matches_independent_matmul():
    wl = synth.WORKLOADS["tiny"]
    p, s, gs = oracle.quantize(synth.weights_f32(wl))
    M = 3
    X = synth.x_bf16_custom(synth.X_NORMAL, M, wl.K)
    x = oracle.bf16_bits_to_f64(X)
    W = independent_dequant(p, s, gs, wl.N, wl.K)
    ref = x @ W.T
    y, ad = oracle.linear(p, s, gs, X, M, wl.N, wl.K)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-15)
    assert np.allclose(ad, np.abs(x)[:, None, :].__mul__(np.abs(W)[None]).sum(-1), rtol=1e-12)


def test_one_hot_selects_one_dequantised_column():
    wl = synth.WORKLOADS["tiny"]
    p, s, gs = oracle.quantize(synth.weights_f32(wl))
    W = independent_dequant(p, s, gs, wl.N, wl.K)
    for k in (0, 1, 17, 255):
        X = np.zeros((1, wl.K), np.uint16)
        X[0, k] = 0x3F80                          # bf16 1.0
        y, _ = oracle.linear(p, s, gs, X, 1, wl.N, wl.K)
        assert np.array_equal(y[0], W[:, k])


def test_brute_force_4x32x16_dyadic():
    """4x32x16 with gs = 1: small-integer X and hand-structured codes; every
    partial sum is a dyadic rational, so the fp64 result is exact."""
    g = grid()
    M, N, K = 4, 32, 16
    codes = np.array([[(n + k) % 16 for k in range(K)] for n in range(N)], np.uint8)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    scodes = np.array([[0x38 if n % 2 == 0 else 0x40] for n in range(N)], np.uint8)  # 1.0 / 2.0
    xs = np.array([[(k % 5) - m for k in range(K)] for m in range(M)], np.float64)
    X = np.array([[torch_bf16_bits(v) for v in row] for row in xs], np.uint16)
    y, _ = oracle.linear(packed, scodes, 1.0, X, M, N, K)
    for m in range(M):
        for n in range(N):
            s = 1.0 if n % 2 == 0 else 2.0
            expect = s * sum(g[(n + k) % 16] * ((k % 5) - m) for k in range(K))
            assert y[m, n] == expect


def test_linear_doubling_and_row_independence():
    wl = synth.WORKLOADS["tiny"]
    p, s, gs = oracle.quantize(synth.weights_f32(wl))
    X = synth.x_bf16_custom(synth.X_NORMAL, 3, wl.K)
    y, _ = oracle.linear(p, s, gs, X, 3, wl.N, wl.K)
    X2 = (X.astype(np.uint32) + 0x0080).astype(np.uint16)     # exponent + 1 = x * 2
    X2[X == 0] = 0
    y2, _ = oracle.linear(p, s, gs, X2, 3, wl.N, wl.K)
    assert np.array_equal(y2, 2 * y)
    for m in range(3):
        ym, _ = oracle.linear(p, s, gs, X[m:m + 1], 1, wl.N, wl.K)
        assert np.array_equal(ym[0], y[m])
    rows = np.array([5, 0, 511, 5])
    yr, _ = oracle.linear(p, s, gs, X, 3, wl.N, wl.K, rows=rows)
    assert np.array_equal(yr, y[:, rows])


def test_count_bad():
    sc = np.array([0x00, 0x7F, 0x7E, 0xFF, 0x80], np.uint8)
    assert oracle.count_bad(sc, 1.0) == 2
    assert oracle.count_bad(sc, float("nan")) == 3
    assert oracle.count_bad(sc, -1.0) == 3
    assert oracle.count_bad(sc, 0.0) == 2


# ----- bytes model --------------------------------------------------------

def test_bytes_model_matches_pages_lm_head():
    d = {k: float(v) for k, v in read_golden("lm_head_bytes.txt")}
    N, K = int(d["rows"]), int(d["cols"])
    nvfp4 = oracle.bytes_model(0, N, K)
    assert nvfp4 == 715_161_600
    assert d["nvfp4_gb_low"] <= nvfp4 / 1e9 <= d["nvfp4_gb_high"] + 0.005
    assert round(N * K * 2 / 1e9, 2) == d["bf16_gb"]
    # X and Y terms: 2*M*K + 2*M*N
    assert oracle.bytes_model(16, N, K) - nvfp4 == 2 * 16 * K + 2 * 16 * N


# ----- epilogues: SwiGLU and greedy argmax / top-k ---------------------------

def _silu_expit(v):
    """SiLU from SciPy's logistic function (independent library code)."""
    from scipy.special import expit
    return np.asarray(v, np.float64) * expit(np.asarray(v, np.float64))


def test_silu_closed_forms():
    assert oracle.silu(0.0) == 0.0
    # sigmoid(ln r) = r / (1 + r) exactly, so silu(ln r) = ln(r) r / (1 + r)
    for r in (0.125, 0.5, 2.0, 3.0, 7.0, 1000.0):
        v = math.log(r)
        assert oracle.silu(v) == pytest.approx(v * r / (1.0 + r), rel=1e-15)
    # odd part: silu(v) - silu(-v) = v
    for v in np.linspace(-30.0, 30.0, 241):
        assert oracle.silu(v) - oracle.silu(-v) == pytest.approx(v, rel=1e-14, abs=1e-300)
    # tails: the limits v and 0
    assert oracle.silu(800.0) == 800.0 and oracle.silu(40.0) == pytest.approx(40.0, rel=1e-16)
    assert oracle.silu(-800.0) == 0.0
    rng = np.random.default_rng(3)
    for v in rng.normal(0.0, 6.0, 200):
        assert oracle.silu(v) == pytest.approx(float(_silu_expit(v)), rel=1e-13, abs=1e-300)


def test_swiglu_pairs_rows_and_gates_with_silu():
    """Against an independent construction: torch/grid decode of W, numpy
    matmul of the even (gate) and odd (up) rows, SciPy's logistic."""
    wl = synth.WORKLOADS["tiny"]
    p, s, gs = oracle.quantize(synth.weights_f32(wl))
    M = 3
    X = synth.x_bf16_custom(synth.X_NORMAL, M, wl.K, seed=4)
    x = oracle.bf16_bits_to_f64(X)
    W = independent_dequant(p, s, gs, wl.N, wl.K)
    g_ref, u_ref = x @ W[0::2].T, x @ W[1::2].T
    h, g, u, adg, adu = oracle.swiglu_linear(p, s, gs, X, M, wl.N, wl.K)
    assert h.shape == (M, wl.N // 2)
    assert np.allclose(g, g_ref, rtol=1e-12, atol=1e-15)
    assert np.allclose(u, u_ref, rtol=1e-12, atol=1e-15)
    assert np.allclose(h, _silu_expit(g_ref) * u_ref, rtol=1e-11, atol=1e-15)
    assert np.allclose(adg, np.abs(x) @ np.abs(W[0::2]).T, rtol=1e-12)
    assert np.allclose(adu, np.abs(x) @ np.abs(W[1::2]).T, rtol=1e-12)
    cols = np.array([255, 0, 7, 7])
    hc, gc, uc, _, _ = oracle.swiglu_linear(p, s, gs, X, M, wl.N, wl.K, cols=cols)
    assert np.array_equal(hc, h[:, cols]) and np.array_equal(gc, g[:, cols])
    assert np.array_equal(uc, u[:, cols])


def test_swiglu_one_hot_exact_values():
    """gs = 1 and X = e_k: gate and up are single decoded weights, and at
    0, +-2688 (= 6 * 448) SiLU is exact in fp64, so h is known exactly."""
    K = 16
    # columns: (gate code, gate scale, up code, up scale) -> h
    table = [(0x0, 0x38, 0x2, 0x38, 0.0),             # gate 0
             (0x7, 0x7E, 0x3, 0x38, 2688.0 * 1.5),    # gate 2688, up 1.5
             (0xF, 0x7E, 0x7, 0x40, -0.0),            # gate -2688: silu = -0
             (0x7, 0x7E, 0x0, 0x38, 0.0)]             # up 0
    N2 = 2 * len(table)
    codes = np.zeros((N2, K), np.uint8)
    sc = np.zeros((N2, 1), np.uint8)
    for c, (gc, gsc, uc, usc, _) in enumerate(table):
        codes[2 * c, :] = gc
        sc[2 * c] = gsc
        codes[2 * c + 1, :] = uc
        sc[2 * c + 1] = usc
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    for k in (0, 5, 15):
        X = np.zeros((1, K), np.uint16)
        X[0, k] = 0x3F80
        h, g, u, _, _ = oracle.swiglu_linear(packed, sc, 1.0, X, 1, N2, K)
        assert [abs(v) for v in h[0]] == [abs(t[4]) for t in table]
        assert g[0, 1] == 2688.0 and g[0, 2] == -2688.0 and u[0, 1] == 1.5


def test_swiglu_tolerance_covers_perturbed_gate_and_up():
    """The derived bound holds for gate and up values perturbed anywhere
    within their own linear bounds, the result rounded to bf16 (torch)."""
    assert oracle.SILU_LIPSCHITZ >= 1.0998
    v = np.linspace(-20.0, 20.0, 400001)
    slope = np.abs(np.diff(_silu_expit(v)) / np.diff(v))
    assert slope.max() <= oracle.SILU_LIPSCHITZ and slope.max() > 1.09
    rng = np.random.default_rng(5)
    n = 4000
    g = rng.uniform(-12.0, 12.0, n)
    u = rng.uniform(-5.0, 5.0, n)
    adg = np.abs(g) * rng.uniform(1.0, 40.0, n)
    adu = np.abs(u) * rng.uniform(1.0, 40.0, n)
    h_ref = _silu_expit(g) * u
    bound = oracle.swiglu_tolerance(h_ref, g, u, adg, adu)
    tg, tu = oracle.tolerance(g, adg), oracle.tolerance(u, adu)
    for sg, su in ((1, 1), (1, -1), (-1, 1), (-1, -1), (None, None)):
        if sg is None:
            dg, du = rng.uniform(-1, 1, n) * tg, rng.uniform(-1, 1, n) * tu
        else:
            dg, du = sg * tg, su * tu
        h = _silu_expit(g + dg) * (u + du)
        hb = torch.tensor(h).to(torch.bfloat16).to(torch.float64).numpy()
        assert np.all(np.abs(hb - h_ref) <= bound)


def test_topk_matches_sorting_bruteforce():
    rng = np.random.default_rng(7)
    y = rng.integers(0, 5, size=(6, 13)).astype(np.float64)   # many ties
    y[5] = 2.0                                                # all equal
    for k in range(1, 14):
        got = oracle.topk(y, k)
        for m in range(y.shape[0]):
            want = sorted(range(y.shape[1]), key=lambda j: (-y[m, j], j))[:k]
            assert list(got[m]) == want, (m, k)
    assert np.array_equal(oracle.topk(y, 1)[:, 0], np.argmax(y, axis=1))  # first maximum
    z = rng.normal(size=(4, 1000))
    assert np.array_equal(oracle.topk(z, 20), np.argsort(-z, axis=1, kind="stable")[:, :20])
    with pytest.raises(ValueError):
        oracle.topk(np.array([[1.0, float("nan")]]), 1)


def test_argmax_decided_uses_both_bounds():
    y = np.array([[1.0, 0.9, 0.0], [1.0, 0.99, 0.0], [0.5, 0.5, 0.1], [0.0, 3.0, 2.0]])
    tol = np.full_like(y, 0.01)
    idx, dec = oracle.argmax_decided(y, tol)
    assert list(idx) == [0, 0, 0, 1]
    assert list(dec) == [True, False, False, True]
    idx1, dec1 = oracle.argmax_decided(np.array([[4.0]]), np.array([[1.0]]))
    assert list(idx1) == [0] and list(dec1) == [True]


# ----- tiers: W4A4 and FP8 weights ----------------------------------------

def _random_nvfp4(rows, K, rng, scale_codes=(0x30, 0x38, 0x40, 0x44)):
    codes = rng.integers(0, 16, size=(rows, K)).astype(np.uint8)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    scales = rng.choice(np.array(scale_codes, np.uint8), size=(rows, K // 16))
    return packed, scales


def test_w4a4_with_x_on_the_grid_equals_the_bf16_linear():
    """gs_x = 1/8: each x_hat = e2m1 * e4m3 / 8 is a bf16 value, so the W4A4
    linear must equal the bf16-X linear on those values, bit for bit."""
    rng = np.random.default_rng(11)
    wl = synth.WORKLOADS["tiny"]
    p, s, gs = oracle.quantize(synth.weights_f32(wl))
    M = 4
    xp, xs = _random_nvfp4(M, wl.K, rng)
    xhat = independent_dequant(xp, xs, 0.125, M, wl.K)
    X = np.array([[torch_bf16_bits(v) for v in row] for row in xhat], np.uint16)
    assert np.array_equal(oracle.bf16_bits_to_f64(X), xhat)      # on the bf16 grid
    y4, ad4 = oracle.linear_w4a4(p, s, gs, xp, xs, 0.125, M, wl.N, wl.K)
    y, ad = oracle.linear(p, s, gs, X, M, wl.N, wl.K)
    assert np.array_equal(y4, y) and np.array_equal(ad4, ad)


def test_w4a4_matches_independent_construction():
    wl = synth.WORKLOADS["tiny"]
    p, s, gs = oracle.quantize(synth.weights_f32(wl))
    M = 3
    X = synth.x_bf16_custom(synth.X_OUTLIERS, M, wl.K, seed=2, n_outliers=4, gain=20.0)
    xp, xs, gs_x = oracle.quantize_x(X)
    x = oracle.bf16_bits_to_f64(X)
    assert gs_x == float(np.float32(np.abs(x).max()) / np.float32(2688.0))
    xhat = independent_dequant(xp, xs, gs_x, M, wl.K)
    W = independent_dequant(p, s, gs, wl.N, wl.K)
    y, ad = oracle.linear_w4a4(p, s, gs, xp, xs, gs_x, M, wl.N, wl.K)
    assert np.allclose(y, xhat @ W.T, rtol=1e-12, atol=1e-15)
    assert np.allclose(ad, np.abs(xhat) @ np.abs(W).T, rtol=1e-12)
    rows = np.array([3, 511, 0])
    yr, _ = oracle.linear_w4a4(p, s, gs, xp, xs, gs_x, M, wl.N, wl.K, rows=rows)
    assert np.array_equal(yr, y[:, rows])
    # each x_hat is within half an E2M1 step of x (steps are <= half the
    # magnitude, or d/2 near zero, d = decoded block scale * gs_x)
    d = np.repeat(np.vectorize(torch_e4m3_value)(xs), 16, axis=1) * gs_x
    assert np.all(np.abs(xhat - x) <= 0.25 * (np.abs(x) + d))


def test_fp8_rows_match_torch_e4m3():
    rng = np.random.default_rng(13)
    w = (rng.normal(0.0, 0.02, size=(64, 96)) * rng.uniform(0.1, 10.0, size=(64, 1))).astype(np.float32)
    w[5] = 0.0
    w[7, 3] = -1e-12                                       # rounds to zero, keeps its sign
    codes, sc = oracle.quantize_fp8_rows(w)
    amax = np.abs(w).max(axis=1)
    assert np.array_equal(sc, amax / np.float32(448.0))
    assert sc[5] == 0.0 and not codes[5].any()
    live = sc > 0
    u = (w[live] / sc[live, None]).astype(np.float32)
    ref = torch.from_numpy(u).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes[live], ref)
    assert codes[7, 3] == 0x80
    with pytest.raises(ValueError):
        oracle.quantize_fp8_rows(np.array([[1.0, float("inf")]], np.float32))


def test_fp8_round_trip_on_grid():
    """Rows of E4M3 values times 2^j that hold +-448 * 2^j quantise back to
    the same codes under s_n = 2^j."""
    rng = np.random.default_rng(17)
    N, K = 16, 64
    codes = rng.integers(1, 0x7F, size=(N, K)).astype(np.uint8)
    codes |= (rng.integers(0, 2, size=(N, K)) << 7).astype(np.uint8)
    codes[:, 0] = 0x7E                                      # 448
    vals = np.vectorize(torch_e4m3_value)(codes)
    pw = 2.0 ** rng.integers(-12, 4, size=(N, 1))
    w = (vals * pw).astype(np.float32)
    got, sc = oracle.quantize_fp8_rows(w)
    assert np.array_equal(sc.astype(np.float64), pw[:, 0])
    assert np.array_equal(got, codes)


def test_fp8_linear_matches_independent_matmul():
    rng = np.random.default_rng(19)
    N, K, M = 40, 128, 3
    w = rng.normal(0.0, 0.05, size=(N, K)).astype(np.float32)
    codes, sc = oracle.quantize_fp8_rows(w)
    X = synth.x_bf16_custom(synth.X_NORMAL, M, K, seed=6)
    x = oracle.bf16_bits_to_f64(X)
    W = np.vectorize(torch_e4m3_value)(codes) * sc.astype(np.float64)[:, None]
    y, ad = oracle.linear_fp8(codes, sc, X, M, N, K)
    assert np.allclose(y, x @ W.T, rtol=1e-12, atol=1e-15)
    assert np.allclose(ad, np.abs(x) @ np.abs(W).T, rtol=1e-12)
    rows = np.array([39, 0, 12])
    yr, _ = oracle.linear_fp8(codes, sc, X, M, N, K, rows=rows)
    assert np.array_equal(yr, y[:, rows])
