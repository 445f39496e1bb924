"""The oracle's pins catch plausible mistakes: each mutant below is the
oracle's source with one planted error (built under the repository's
git-ignored _build/ folder, never into the package), and at least one pin of
tests/test_oracle_pins.py must fail against it. The unmutated oracle passes them all (that module).

Runs on the CPU only; the GPU path is not involved."""
import inspect
import os
import subprocess

import pytest

import oracle
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "nvfp4_oracle.cpp")
BUILD = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "_build", "oracle_mutants")

# name -> (text in the oracle source, replacement); each text occurs exactly once
MUTANTS = {
    "nibble order swapped when packing": (
        "out[j / 2] = uint8_t(q0 | (q1 << 4));",
        "out[j / 2] = uint8_t(q1 | (q0 << 4));"),
    "wrong scale block index in the linear": (
        "ora_e4m3_decode(scales[n * (K / 16) + k / 16]) * double(gs);",
        "ora_e4m3_decode(scales[n * (K / 16) + k / 32]) * double(gs);"),
    "E2M1 sign dropped": (
        "double mag = (e == 0) ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, int(e) - 1);\n  return s ? -mag : mag;",
        "double mag = (e == 0) ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, int(e) - 1);\n  return mag;"),
    "block scale divides by 4 instead of 6": (
        "float t = amax_b / 6.0f;",
        "float t = amax_b / 4.0f;"),
    "ties rounded away from zero": (
        "return (lo % 2 == 0) ? lo : hi;",
        "return hi;"),
    "X indexed transposed": (
        "double p = wrow[size_t(k)] * xm[k];",
        "double p = wrow[size_t(k)] * x[size_t(k * M + m) % size_t(M * K)];"),
    "SiLU gate sign flipped": (
        "return v / (1.0 + std::exp(-v));",
        "return v / (1.0 + std::exp(v));"),
    "gate and up rows swapped": (
        "rows[size_t(c)] = 2 * col;                 // gate rows first ...\n"
        "    rows[size_t(ncols + c)] = 2 * col + 1;",
        "rows[size_t(c)] = 2 * col + 1;\n"
        "    rows[size_t(ncols + c)] = 2 * col;"),
    "top-k ties to the highest index": (
        "(row[a] == row[b] && a < b)",
        "(row[a] == row[b] && a > b)"),
    "W4A4 drops the activation scale": (
        "ora_dequant_f64(x_packed, x_scales, gs_x, M, K, xhat.data());",
        "ora_dequant_f64(x_packed, x_scales, 1.0f, M, K, xhat.data());"),
    "FP8 row scale over 256 instead of 448": (
        "const float sn = amax / 448.0f;",
        "const float sn = amax / 256.0f;"),
    "FP8 linear drops the row scale": (
        "ora_e4m3_decode(codes[n * K + k]) * sn * xv[size_t(m * K + k)];",
        "ora_e4m3_decode(codes[n * K + k]) * xv[size_t(m * K + k)];"),
    "last product of each row dropped": (
        "for (int64_t k = 0; k < K; ++k) {\n          double p",
        "for (int64_t k = 0; k < K - 1; ++k) {\n          double p"),
}

PIN_TESTS = [(name, fn) for name, fn in sorted(vars(pins).items())
             if name.startswith("test_") and callable(fn) and not inspect.signature(fn).parameters]


def _build_mutant(tag, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation site must be unique: %r" % old
    os.makedirs(BUILD, exist_ok=True)
    path = os.path.join(BUILD, "mutant_%s_%d.cpp" % (tag, os.getpid()))
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = path[:-4] + ".so"
    subprocess.run(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-shared",
                    "-fPIC", "-pthread", "-I", os.path.dirname(SRC), "-o", str(lib), str(path)],
                   check=True)
    return str(lib)


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_catch_planted_mistake(mutant, monkeypatch):
    lib = _build_mutant("%d" % sorted(MUTANTS).index(mutant), *MUTANTS[mutant])
    monkeypatch.setattr(oracle, "build", lambda force=False: lib)
    monkeypatch.setattr(oracle, "_lib", None)
    caught = []
    try:
        for name, fn in PIN_TESTS:
            try:
                fn()
            except Exception:            # an assertion or a rejected result
                caught.append(name)
    finally:
        oracle._lib = None               # the next user reloads the real oracle
        for f in (lib, lib[:-3] + ".cpp"):
            if os.path.exists(f):
                os.remove(f)
    assert caught, "no pin fails for mutant: %s" % mutant
