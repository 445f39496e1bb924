"""The seeded input generators: determinism, counter-based indexing, recipes."""
import math

import numpy as np

import synth


def mix64(z):
    z &= (1 << 64) - 1
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & ((1 << 64) - 1)
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & ((1 << 64) - 1)
    return z ^ (z >> 31)


def test_splitmix64_published_definition():
    # The draw of stream (seed, id) at index i is mix(key + (i+1) * gamma).
    gamma = 0x9E3779B97F4A7C15
    for seed, sid in [(0, 0), (0, 1), (7, 103)]:
        key = mix64(mix64(seed) ^ ((sid * 0xD1B54A32D192ED03) & ((1 << 64) - 1)))
        for i in (0, 1, 5, 1 << 40):
            assert synth.draw(seed, sid, i) == mix64(key + (i + 1) * gamma)


def test_splitmix64_reference_sequence():
    # With state 0 the sequential SplitMix64 generator's first outputs are the
    # published test values (state += gamma, then mix).
    gamma = 0x9E3779B97F4A7C15
    outs = [mix64((i + 1) * gamma) for i in range(3)]
    assert outs[0] == 0xE220A8397B1DCDAF
    assert outs[1] == 0x6E789E6AA1B965F4
    assert outs[2] == 0x06C45D188009454F


def test_counter_based_slices_agree():
    wl = synth.WORKLOADS["tiny"]
    full = synth.weights_f32(wl)
    part = synth.weights_f32(wl, rows=slice(100, 140))
    assert np.array_equal(full[100:140], part)
    assert np.array_equal(full, synth.weights_f32(wl))          # deterministic
    assert not np.array_equal(full, synth.weights_f32(wl, copy=1))


def test_normal_moments():
    z = synth.normal_f32(1 << 20, sigma=0.02)
    assert abs(z.mean()) < 1e-4
    assert abs(z.std() - 0.02) < 1e-4


def test_outlier_channels():
    wl = synth.WORKLOADS["decode"]
    idx = synth.distinct_indices(wl.K, 8)
    assert len(set(idx.tolist())) == 8 and idx.min() >= 0 and idx.max() < wl.K
    X = synth.x_bf16(wl, 2)
    x = (X.astype(np.uint32) << 16).view(np.float32)
    base = (synth.x_bf16_custom(synth.X_NORMAL, 2, wl.K).astype(np.uint32) << 16).view(np.float32)
    mask = np.zeros(wl.K, bool)
    mask[idx] = True
    assert np.array_equal(x[:, ~mask], base[:, ~mask])
    ratio = x[:, mask] / base[:, mask]
    assert np.all(np.abs(ratio - 20) < 0.2)


def test_swiglu_and_rmsnorm_recipes():
    wl = synth.WORKLOADS["down"]
    X = synth.x_bf16(wl, 1)
    x = (X.astype(np.uint32) << 16).view(np.float32).astype(np.float64)[0]
    a = np.array([synth.normal(0, 3, i) for i in range(64)])
    b = np.array([synth.normal(0, 4, i) for i in range(64)])
    ref = a / (1 + np.exp(-a)) * b
    assert np.allclose(x[:64], ref, rtol=1e-2, atol=1e-3)
    wl = synth.WORKLOADS["lm_head"]
    X = synth.x_bf16(wl, 2)
    x = (X.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    rms = np.sqrt((x ** 2).mean(axis=1))
    assert np.all(np.abs(rms - 1) < 1e-2)


def test_workload_shapes():
    W = synth.WORKLOADS
    assert (W["decode"].K, W["decode"].N) == (5120, 34816)
    assert W["verify"].Ms == (1, 2, 4, 8, 12, 16)
    assert (W["down"].K, W["down"].N, W["down"].copies) == (17408, 5120, 64)
    assert (W["lm_head"].K, W["lm_head"].N) == (5120, 248320)
    assert math.isclose(W["down"].w_sigma, 0.02 / math.sqrt(3.4))
