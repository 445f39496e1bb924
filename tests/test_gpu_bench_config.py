"""Parity in the launch configuration bench.py times: CUDA graphs of 64
back-to-back calls with programmatic dependent launch, rotated weight copies
larger than L2. Y after the timed replays is checked against the oracle on
sampled rows. The oracle quantises the workload's weights itself (the bench
quantises on the GPU; both quantisers are checked bit-identical elsewhere)."""
import numpy as np
import pytest
import torch

import bench
import nvfp4_weight_streaming_b200 as nv
import oracle
import synth
from tests.gpu_util import check_tolerance, host_u16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,M", [("decode", 1), ("verify", 16)])
def test_bench_launch_configuration_matches_oracle(name, M):
    wl = synth.WORKLOADS[name]
    l2 = getattr(torch.cuda.get_device_properties(0), "L2_cache_size", 126 * 2 ** 20)
    pb = bench.Problem(name, M, nv.NVFP4_VARIANT_AUTO, min_footprint=4.2 * l2, flags=nv.NVFP4_PLAN_PDL)
    try:
        bench.time_problem(pb, 128, 3, 1)
        pb.check_status()
        y = host_u16(pb.y).reshape(M, wl.N)
    finally:
        pb.destroy()
    packed, scales, gs = oracle.quantize(synth.weights_f32(wl))
    rows = np.arange(0, wl.N, 61)
    y_ref, ad = oracle.linear(packed, scales, gs, synth.x_bf16(wl, M), M, wl.N, wl.K, rows=rows)
    check_tolerance(y[:, rows], y_ref, ad)
