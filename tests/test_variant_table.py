"""The AUTO variant choice: a table of measured per-variant times compiled
into the library. Host tests check that the compiled table is the one the
committed measurements give, that every measured shape gets its fastest
variant, and the nearest-shape rule elsewhere; a GPU test checks that plans
follow the choice and fall back when the chosen variant cannot take a plan.
"""
import csv
import math
import os
import random

import pytest

import nvfp4_weight_streaming_b200 as nv
from nvfp4_weight_streaming_b200 import gen_variant_table

CSV = os.path.join(os.path.dirname(nv.__file__), "csrc", "variant_table.csv")
COLS = {"gemv_us": nv.NVFP4_VARIANT_GEMV, "mma_us": nv.NVFP4_VARIANT_MMA,
        "tc_us": nv.NVFP4_VARIANT_TC, "row_us": nv.NVFP4_VARIANT_ROW}


def measured():
    with open(CSV) as f:
        lines = [ln for ln in f if ln.strip() and not ln.startswith("#")]
    rows = []
    for rec in csv.DictReader(lines):
        times = {COLS[k]: float(v) for k, v in rec.items() if k in COLS and v}
        rows.append((int(rec["M"]), int(rec["N"]), int(rec["K"]), times))
    return rows


def test_table_covers_the_workload_shapes():
    shapes = {(M, N, K) for M, N, K, _ in measured()}
    for M in (1, 2, 4, 8, 12, 16):
        assert (M, 34816, 5120) in shapes
    for M in (1, 4, 8, 16):
        assert (M, 5120, 17408) in shapes
    for M in (1, 8, 16):
        assert (M, 248320, 5120) in shapes
    assert (1, 512, 256) in shapes
    # every row has the MMA time and at least one other variant to compare with
    for M, N, K, times in measured():
        assert nv.NVFP4_VARIANT_MMA in times and len(times) >= 2, (M, N, K)


def test_compiled_table_is_generated_from_the_measurements():
    inc = os.path.join(os.path.dirname(CSV), "variant_table.inc")
    assert open(inc).read() == gen_variant_table.render(gen_variant_table.read(CSV))


def test_measured_shapes_get_their_fastest_variant():
    for M, N, K, times in measured():
        best = min(times, key=lambda v: times[v])
        assert nv.nvfp4_auto_variant(M, N, K) == best, (M, N, K, times)


def _nearest(M, N, K, rows):
    best, v = None, None
    for Mt, Nt, Kt, times in rows:
        d = 2 * abs(math.log2(M) - math.log2(Mt)) + abs(math.log2(N * K) - math.log2(Nt * Kt))
        if best is None or d < best:
            best, v = d, min(times, key=lambda x: times[x])
    return v


def test_other_shapes_take_the_nearest_measured_shape():
    rows = measured()
    rnd = random.Random(7)
    for _ in range(300):
        M = rnd.randint(1, 16)
        N = rnd.randint(1, 300000)
        K = 256 * rnd.randint(1, 80)
        assert nv.nvfp4_auto_variant(M, N, K) == _nearest(M, N, K, rows), (M, N, K)


def test_auto_variant_argument_errors():
    for args in [(0, 16, 256), (17, 16, 256), (1, -1, 256), (1, 16, -256), (1, 16, 100)]:
        assert nv.nvfp4_auto_variant(*args) == -1


@pytest.mark.gpu
def test_plans_follow_the_table_and_fall_back():
    import torch
    d = torch.cuda.current_device()
    for M, N, K, times in measured():
        want = min(times, key=lambda v: times[v])
        p = nv.nvfp4_linear_plan(M, N, K, d, nv.NVFP4_VARIANT_AUTO)
        try:
            assert nv.nvfp4_linear_variant(p) == want, (M, N, K)
        finally:
            nv.nvfp4_linear_destroy(p)
    # a GEMV shape with a fused epilogue: the epilogues live in the MMA variant
    assert nv.nvfp4_auto_variant(1, 1024, 1024) == nv.NVFP4_VARIANT_GEMV
    p = nv.nvfp4_linear_plan(1, 1024, 1024, d, nv.NVFP4_PLAN_EPI_SWIGLU)
    try:
        assert nv.nvfp4_linear_variant(p) == nv.NVFP4_VARIANT_MMA
    finally:
        nv.nvfp4_linear_destroy(p)
