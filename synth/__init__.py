"""Seeded synthetic inputs for the NVFP4 weight-streaming linear.

A module of its own: the oracle's callers (tests) and the benchmark both draw
their inputs here. It contains no arithmetic of the linear itself (no
quantisation, decode or contraction) -- only random numbers and the input
recipes below. The generator is SplitMix64 used counter-style plus Box-Muller
(see synth.cpp), so any element can be drawn on its own.

Workloads (shapes of a 27B-class decoder with hidden size 5120 and a
248,320-entry vocabulary; page "Qwen3.8-27B-NVFP4-RTX5090 API & Inference
Endpoint", section "Why lm_head is NVFP4, and why MTP is gone"):

  tiny     M=1,  K=256,   N=512      W~N(0,0.02)            X~N(0,1)
  decode   M=1,  K=5120,  N=34816    W~N(0,0.02)            X~N(0,1), 8 channels x20
  verify   M in {1,2,4,8,12,16}, same weights and X recipe as decode
  down     K=17408, N=5120, M in {1,4,8,16}  W~N(0,0.02/sqrt(3.4))  X=SiLU(a)*b
  lm_head  K=5120, N=248320, M in {1,8,16}   W~N(0,0.01)   X RMS-normalised N(0,1)

Streams: W copy 0 = stream 0, copy c >= 1 = stream 100+c; X = stream 1;
outlier channels = stream 2; SiLU inputs a, b = streams 3, 4. Seed 0.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.cpp")
_LIB = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_lib = None
# host threads: the cores this process may run on (its affinity mask), which
# can be fewer than the machine's
NTHREADS = max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity")
               else (os.cpu_count() or 1))

X_NORMAL, X_OUTLIERS, X_SWIGLU, X_RMSNORM = 0, 1, 2, 3


@dataclass(frozen=True)
class Workload:
    name: str
    K: int
    N: int
    Ms: tuple
    w_sigma: float
    x_kind: int
    copies: int = 1
    n_outliers: int = 0
    outlier_gain: float = 1.0
    seed: int = 0


WORKLOADS = {
    "tiny": Workload("tiny", 256, 512, (1,), 0.02, X_NORMAL),
    "decode": Workload("decode", 5120, 34816, (1,), 0.02, X_OUTLIERS,
                       n_outliers=8, outlier_gain=20.0),
    "verify": Workload("verify", 5120, 34816, (1, 2, 4, 8, 12, 16), 0.02, X_OUTLIERS,
                       n_outliers=8, outlier_gain=20.0),
    "down": Workload("down", 17408, 5120, (1, 4, 8, 16), 0.02 / math.sqrt(3.4), X_SWIGLU,
                     copies=64),
    "lm_head": Workload("lm_head", 5120, 248320, (1, 8, 16), 0.01, X_RMSNORM),
}


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.run(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread",
                        "-o", tmp, _SRC], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            c = ctypes
            lib.synth_draw.restype = c.c_uint64
            lib.synth_draw.argtypes = [c.c_uint64, c.c_uint64, c.c_uint64]
            lib.synth_uniform.restype = c.c_double
            lib.synth_uniform.argtypes = [c.c_uint64, c.c_uint64, c.c_uint64]
            lib.synth_normal.restype = c.c_double
            lib.synth_normal.argtypes = [c.c_uint64, c.c_uint64, c.c_uint64]
            lib.synth_normal_f32.restype = None
            lib.synth_normal_f32.argtypes = [c.c_uint64, c.c_uint64, c.c_uint64, c.c_int64,
                                             c.c_double, c.c_void_p, c.c_int]
            lib.synth_distinct_indices.restype = c.c_int
            lib.synth_distinct_indices.argtypes = [c.c_uint64, c.c_uint64, c.c_int64,
                                                   c.c_int64, c.c_void_p]
            lib.synth_x_bf16.restype = c.c_int
            lib.synth_x_bf16.argtypes = [c.c_int, c.c_uint64, c.c_int64, c.c_int64, c.c_int64,
                                         c.c_double, c.c_void_p]
            _lib = lib
        return _lib


def draw(seed: int, stream: int, i: int) -> int:
    return int(_load().synth_draw(seed, stream, i))


def uniform(seed: int, stream: int, i: int) -> float:
    return float(_load().synth_uniform(seed, stream, i))


def normal(seed: int, stream: int, i: int) -> float:
    return float(_load().synth_normal(seed, stream, i))


def normal_f32(n: int, sigma: float = 1.0, seed: int = 0, stream: int = 0, start: int = 0,
               out: np.ndarray | None = None, nthreads: int = NTHREADS) -> np.ndarray:
    if out is None:
        out = np.empty(n, np.float32)
    assert out.dtype == np.float32 and out.flags.c_contiguous and out.size == n
    _load().synth_normal_f32(seed, stream, start, n, float(sigma), out.ctypes.data, nthreads)
    return out


def weight_stream(copy: int) -> int:
    return 0 if copy == 0 else 100 + copy


def weights_f32(wl: Workload, copy: int = 0, rows: slice | None = None,
                nthreads: int = NTHREADS) -> np.ndarray:
    """fp32 W [N][K] (or the row range `rows`) of workload wl, copy `copy`."""
    r0, r1 = (0, wl.N) if rows is None else (rows.start or 0, rows.stop if rows.stop is not None else wl.N)
    out = np.empty((r1 - r0, wl.K), np.float32)
    normal_f32(out.size, wl.w_sigma, wl.seed, weight_stream(copy), start=r0 * wl.K,
               out=out.reshape(-1), nthreads=nthreads)
    return out


def distinct_indices(K: int, count: int, seed: int = 0, stream: int = 2) -> np.ndarray:
    out = np.zeros(count, np.int64)
    if _load().synth_distinct_indices(seed, stream, K, count, out.ctypes.data):
        raise ValueError("bad arguments")
    return out


def x_bf16(wl: Workload, M: int) -> np.ndarray:
    """Activations X [M][K] of workload wl as bf16 bit patterns (uint16)."""
    out = np.empty((M, wl.K), np.uint16)
    rc = _load().synth_x_bf16(wl.x_kind, wl.seed, M, wl.K, wl.n_outliers, wl.outlier_gain,
                              out.ctypes.data)
    if rc:
        raise ValueError("synth_x_bf16 failed")
    return out


def x_bf16_custom(kind: int, M: int, K: int, seed: int = 0, n_outliers: int = 0,
                  gain: float = 1.0) -> np.ndarray:
    out = np.empty((M, K), np.uint16)
    if _load().synth_x_bf16(kind, seed, M, K, n_outliers, gain, out.ctypes.data):
        raise ValueError("synth_x_bf16 failed")
    return out
