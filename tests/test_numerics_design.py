"""The numerical facts the kernels' design rests on, checked on the CPU with
numpy's IEEE float16/float32 arithmetic (round to nearest even, subnormals
kept). These test the arguments, not the kernels; the GPU parity tests test
the kernels.

1. Every product e2m1(code) * e4m3(scale) of a finite scale is exact in f16,
   so the weight operand of the f16 MMA carries no rounding (format: page
   "Qwen3.8-27B-NVFP4-RTX5090 API & Inference Endpoint", section "Recipe
   (NVIDIA ModelOpt)": NVFP4 with 16-element E4M3 scale groups).
2. A bf16 row of X, shifted by the power of two that puts its largest
   magnitude in [2^14, 2^15), splits into an f16 hi plane plus an f16 lo plane
   scaled by 2^29 that reproduces every element exactly down to 2^57 below the
   row maximum; smaller elements are off by at most 2^-54 of the shifted unit.
3. The product of two f16 values is exact in fp32 (11 + 11 significant bits),
   so an MMA with f32 accumulation rounds only in its sums.
"""
import numpy as np

from tests.conftest import read_golden

LO_SHIFT = 29


def _grid():
    return {int(c): float(v) for c, v in read_golden("e2m1_grid.txt")}


def _e4m3_finite_values():
    import torch
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    v = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return v[np.isfinite(v)]


def test_e2m1_times_e4m3_products_exact_in_f16():
    g = np.array(list(_grid().values()))
    s = _e4m3_finite_values()
    assert s.size == 254
    prod = np.multiply.outer(g, s).ravel()             # exact in fp64
    assert np.array_equal(prod.astype(np.float16).astype(np.float64), prod)
    assert np.abs(prod).max() == 2688.0 and np.abs(prod).max() < np.finfo(np.float16).max


def _bf16_to_f32(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32)


def split_row(bits):
    """hi, lo planes (float16) and the shift sh of one bf16 row, following the
    argument: sh = 14 - floor(log2 max|x|), s = x * 2^sh in fp32 (applied as
    two powers of two), hi = f16(s), lo = f16((s - hi) * 2^29)."""
    x = _bf16_to_f32(bits)
    mag = float(np.abs(x).max()) if x.size else 0.0
    if mag == 0.0:
        sh = 0
    else:
        _, e = np.frexp(mag)                            # mag = f * 2^e, f in [0.5, 1)
        sh = 14 - (int(e) - 1)
    h1 = int(sh / 2)                                    # truncation toward zero
    f1, f2 = np.float32(2.0 ** h1), np.float32(2.0 ** (sh - h1))
    s = (x * f1) * f2
    hi = s.astype(np.float16)
    lo = ((s - hi.astype(np.float32)) * np.float32(2.0 ** LO_SHIFT)).astype(np.float16)
    return hi, lo, sh


def _random_bf16_row(rng, K, span):
    """Normals times 2^U(-span, 0), rounded to bf16 (nearest even) as bits."""
    v = rng.normal(size=K) * np.exp2(rng.uniform(-span, 0.0, size=K))
    v = v.astype(np.float32).view(np.uint32)
    r = ((v >> 16) & 1) + 0x7FFF
    return ((v + r) >> 16).astype(np.uint16)


def _check_row(bits):
    hi, lo, sh = split_row(bits)
    x = _bf16_to_f32(bits).astype(np.float64)
    s_exact = np.ldexp(x, sh)                           # exact in fp64 for these ranges
    recon = hi.astype(np.float64) + np.ldexp(lo.astype(np.float64), -LO_SHIFT)
    err = np.abs(recon - s_exact)
    mag = np.abs(x).max()
    if mag == 0.0:
        assert not err.any()
        return
    assert 2.0 ** 14 <= np.abs(s_exact).max() < 2.0 ** 15
    assert np.abs(hi.astype(np.float64)).max() < 2.0 ** 15          # no f16 overflow
    big = np.abs(s_exact) >= 2.0 ** (14 - 57)
    assert not err[big].any(), "an element within 2^57 of the maximum was not exact"
    assert np.all(err <= 2.0 ** -54)


def test_hi_lo_planes_reproduce_bf16_rows():
    rng = np.random.default_rng(23)
    for span in (4.0, 20.0, 60.0, 90.0, 140.0):
        for _ in range(20):
            _check_row(_random_bf16_row(rng, 512, span))


def test_hi_lo_planes_edge_rows():
    rng = np.random.default_rng(29)
    _check_row(np.zeros(64, np.uint16))                 # all zero: nothing to scale
    row = _random_bf16_row(rng, 64, 8.0)
    row[3] = 0x7F7F                                      # largest finite bf16 (~3.39e38)
    row[7] = 0x0001                                      # smallest subnormal (2^-133)
    _check_row(row)
    tiny = np.full(64, 0x0001, np.uint16)               # a row of subnormals
    tiny[5] = 0x0040
    _check_row(tiny)
    neg = _random_bf16_row(rng, 64, 30.0) | np.uint16(0x8000)
    _check_row(neg)


def test_f16_products_exact_in_f32():
    rng = np.random.default_rng(31)
    a = rng.normal(size=20000).astype(np.float16)
    b = (rng.normal(size=20000) * 1e3).astype(np.float16)
    prod64 = a.astype(np.float64) * b.astype(np.float64)
    prod32 = a.astype(np.float32) * b.astype(np.float32)
    assert np.array_equal(prod32.astype(np.float64), prod64)


def _make_f16_rn(sign, t, sig):
    """The integer rounding of the tcgen05 variant's lo plane, restated: the
    f16 bits of sign * sig/128 * 2^t (sig in [128, 255]) rounded to nearest
    even, subnormals included."""
    if t >= -14:
        return (sign << 15) | ((t + 15) << 10) | ((sig & 0x7F) << 3)
    sh = t + 17
    if sh >= 0:
        q = sig << sh
    else:
        n = -sh
        if n > 9:
            return sign << 15
        half, rest = 1 << (n - 1), sig & ((1 << n) - 1)
        q = sig >> n
        if rest > half or (rest == half and (q & 1)):
            q += 1
    return (sign << 15) | q


def test_integer_f16_rounding_matches_ieee():
    """Every significand at every exponent from 2^15 down past the last f16
    subnormal: the integer rounding equals IEEE round-to-nearest-even."""
    for t in range(-45, 16):
        for sig in range(128, 256):
            for sign in (0, 1):
                v = (-1.0 if sign else 1.0) * sig / 128.0 * 2.0 ** t
                ref = int(np.array([v], np.float16).view(np.uint16)[0])
                assert _make_f16_rn(sign, t, sig) == ref, (sign, t, sig)
