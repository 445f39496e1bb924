"""CPU oracle for the NVFP4 weight-streaming linear -- TEST INFRASTRUCTURE ONLY.

Only tests/, the smoke check in __graft_entry__ and the CPU-baseline leg of
bench.py may import this package. The product (nvfp4_weight_streaming_b200)
never imports it and shares no code with it.

The arithmetic lives in nvfp4_oracle.cpp (plain host C++, fp64 accumulation);
this module only compiles it (g++) and marshals numpy arrays through ctypes.
Every function cites, in the C++ source, the passage it follows:
  * "Qwen3.8-27B-NVFP4-RTX5090 API & Inference Endpoint", section "Recipe
    (NVIDIA ModelOpt)": NVFP4 with 16-element groups; section "Serving": the
    4-bit codes are stored packed in uint8 tensors.
  * "InventDB Sparkle", section "How it answers quickly": the weight read per
    token and the one-pass check of drafted tokens (M = 1..16).
  * "SparkInfer" README, sections "Layout & scoring" (fused FFN kernels) and
    "DSpark speculative decode" (greedy decoding); "Qwen3.8-27B-NVFP4-RTX5090
    API & Inference Endpoint", section "SparkInfer + DSpark" (near ties at the
    top of the logits): the SwiGLU and argmax / top-k epilogues.
  * "Qwen3.8-27B-NVFP4-RTX5090 API & Inference Endpoint", section "Recipe
    (NVIDIA ModelOpt)" (W4A4, group size 16, per-layer input scale) and
    "InventDB Sparkle", section "How it answers quickly" (8-bit weights): the
    W4A4 and FP8 weight tiers.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.cpp")
_HDR = os.path.join(_HERE, "nvfp4_oracle.h")
_LIB = os.path.join(_HERE, "libnvfp4_oracle.so")
_lock = threading.Lock()
_lib = None

# host threads: the cores this process may run on (its affinity mask), which
# can be fewer than the machine's
NTHREADS = max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity")
               else (os.cpu_count() or 1))


def build(force: bool = False) -> str:
    """Compile the oracle library in place (host g++); returns its path."""
    stale = (not os.path.exists(_LIB) or
             os.path.getmtime(_LIB) < max(os.path.getmtime(_SRC), os.path.getmtime(_HDR)))
    if force or stale:
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-pthread", "-o", tmp, _SRC]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        c = ctypes
        P = c.c_void_p
        sig = {
            "ora_threads_for": (c.c_int, [c.c_int64, c.c_int]),
            "ora_e2m1_decode": (c.c_double, [c.c_uint32]),
            "ora_e4m3_decode": (c.c_double, [c.c_uint32]),
            "ora_e4m3_is_nan": (c.c_int, [c.c_uint32]),
            "ora_e2m1_encode": (c.c_uint32, [c.c_float]),
            "ora_e4m3_encode": (c.c_uint32, [c.c_float]),
            "ora_global_scale": (c.c_int, [P, c.c_int64, P, c.c_int]),
            "ora_quantize_rows": (c.c_int, [P, c.c_int64, c.c_int64, c.c_float, P, P, c.c_int]),
            "ora_quantize": (c.c_int, [P, c.c_int64, c.c_int64, P, P, P, c.c_int]),
            "ora_dequant_f64": (c.c_int, [P, P, c.c_float, c.c_int64, c.c_int64, P]),
            "ora_dequant_bf16_nogs": (c.c_int, [P, P, c.c_int64, c.c_int64, P]),
            "ora_count_bad": (c.c_int64, [P, c.c_int64, c.c_float]),
            "ora_linear": (c.c_int, [P, P, c.c_float, P, c.c_int64, c.c_int64, c.c_int64,
                                     P, c.c_int64, P, P, c.c_int]),
            "ora_silu": (c.c_double, [c.c_double]),
            "ora_swiglu_linear": (c.c_int, [P, P, c.c_float, P, c.c_int64, c.c_int64, c.c_int64,
                                            P, c.c_int64, P, P, P, P, P, c.c_int]),
            "ora_topk": (c.c_int, [P, c.c_int64, c.c_int64, c.c_int64, P]),
            "ora_linear_w4a4": (c.c_int, [P, P, c.c_float, P, P, c.c_float, c.c_int64, c.c_int64,
                                          c.c_int64, P, c.c_int64, P, P, c.c_int]),
            "ora_quantize_fp8_rows": (c.c_int, [P, c.c_int64, c.c_int64, P, P, c.c_int]),
            "ora_linear_fp8": (c.c_int, [P, P, P, c.c_int64, c.c_int64, c.c_int64, P, c.c_int64,
                                         P, P, c.c_int]),
            "ora_bf16_rne": (c.c_uint16, [c.c_double]),
            "ora_bf16_value": (c.c_double, [c.c_uint16]),
            "ora_bytes_model": (c.c_double, [c.c_int64, c.c_int64, c.c_int64]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def threads_for(nrows: int, nthreads: int = NTHREADS) -> int:
    """Host threads the row-parallel oracle functions use for `nrows` rows."""
    return int(_load().ora_threads_for(int(nrows), int(nthreads)))


# ---- scalar codecs -------------------------------------------------------

def e2m1_decode(code: int) -> float:
    return _load().ora_e2m1_decode(int(code))


def e4m3_decode(code: int) -> float:
    return _load().ora_e4m3_decode(int(code))


def e4m3_is_nan(code: int) -> bool:
    return bool(_load().ora_e4m3_is_nan(int(code)))


def e2m1_encode(r: float) -> int:
    return int(_load().ora_e2m1_encode(float(np.float32(r))))


def e4m3_encode(u: float) -> int:
    return int(_load().ora_e4m3_encode(float(np.float32(u))))


def bf16_rne(v: float) -> int:
    return int(_load().ora_bf16_rne(float(v)))


def bf16_value(bits: int) -> float:
    return _load().ora_bf16_value(int(bits))


def bytes_model(M: int, N: int, K: int) -> float:
    return _load().ora_bytes_model(M, N, K)


# ---- array routines -------------------------------------------------------

def global_scale(w: np.ndarray, nthreads: int = NTHREADS) -> float:
    w = _c(w, np.float32)
    gs = np.zeros(1, np.float32)
    rc = _load().ora_global_scale(_ptr(w), w.size, _ptr(gs), nthreads)
    if rc:
        raise ValueError("ora_global_scale failed (%d)" % rc)
    return float(gs[0])


def quantize(w: np.ndarray, nthreads: int = NTHREADS):
    """w: fp32 [N][K] -> (packed u8 [N][K/2], scales u8 [N][K/16], gs float)."""
    w = _c(w, np.float32)
    N, K = w.shape
    packed = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, K // 16), np.uint8)
    gs = np.zeros(1, np.float32)
    rc = _load().ora_quantize(_ptr(w), N, K, _ptr(packed), _ptr(scales), _ptr(gs), nthreads)
    if rc:
        raise ValueError("ora_quantize failed (%d)" % rc)
    return packed, scales, float(gs[0])


def quantize_rows(w: np.ndarray, gs: float, nthreads: int = NTHREADS):
    w = _c(w, np.float32)
    N, K = w.shape
    packed = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, K // 16), np.uint8)
    rc = _load().ora_quantize_rows(_ptr(w), N, K, float(gs), _ptr(packed), _ptr(scales), nthreads)
    if rc:
        raise ValueError("ora_quantize_rows failed (%d)" % rc)
    return packed, scales


def dequant_f64(packed, scales, gs, N, K) -> np.ndarray:
    packed = _c(packed, np.uint8)
    scales = _c(scales, np.uint8)
    out = np.zeros((N, K), np.float64)
    rc = _load().ora_dequant_f64(_ptr(packed), _ptr(scales), float(gs), N, K, _ptr(out))
    if rc:
        raise ValueError("ora_dequant_f64 failed (%d)" % rc)
    return out


def dequant_bf16_nogs(packed, scales, N, K) -> np.ndarray:
    packed = _c(packed, np.uint8)
    scales = _c(scales, np.uint8)
    out = np.zeros((N, K), np.uint16)
    rc = _load().ora_dequant_bf16_nogs(_ptr(packed), _ptr(scales), N, K, _ptr(out))
    if rc:
        raise ValueError("ora_dequant_bf16_nogs failed (%d)" % rc)
    return out


def count_bad(scales, gs) -> int:
    scales = _c(scales, np.uint8)
    return int(_load().ora_count_bad(_ptr(scales), scales.size, float(gs)))


def linear(packed, scales, gs, x_bf16, M, N, K, rows=None, nthreads: int = NTHREADS):
    """Reference linear. Returns (y fp64 [M][nrows], absdot fp64 [M][nrows])."""
    packed = _c(packed, np.uint8)
    scales = _c(scales, np.uint8)
    x_bf16 = _c(x_bf16, np.uint16)
    if rows is None:
        nrows = N
        rows_arr = None
    else:
        rows_arr = _c(rows, np.int64)
        nrows = rows_arr.size
    y = np.zeros((M, nrows), np.float64)
    ad = np.zeros((M, nrows), np.float64)
    rc = _load().ora_linear(_ptr(packed), _ptr(scales), float(gs), _ptr(x_bf16), M, N, K,
                            _ptr(rows_arr), nrows, _ptr(y), _ptr(ad), nthreads)
    if rc:
        raise ValueError("ora_linear failed (%d)" % rc)
    return y, ad


def tolerance(y_ref: np.ndarray, absdot: np.ndarray) -> np.ndarray:
    """Per-element bound |y - y_ref| <= 1e-2 |y_ref| + 1e-4 sum_k |w_hat x|."""
    return 1e-2 * np.abs(y_ref) + 1e-4 * absdot


def silu(v: float) -> float:
    return float(_load().ora_silu(float(v)))


def swiglu_linear(packed, scales, gs, x_bf16, M, N2, K, cols=None, nthreads: int = NTHREADS):
    """SiLU-gated output of a fused gate+up projection (rows 2c, 2c+1 = gate,
    up of output column c). Returns (h, gate, up, absdot_gate, absdot_up),
    each fp64 [M][ncols]."""
    packed = _c(packed, np.uint8)
    scales = _c(scales, np.uint8)
    x_bf16 = _c(x_bf16, np.uint16)
    if cols is None:
        ncols = N2 // 2
        cols_arr = None
    else:
        cols_arr = _c(cols, np.int64)
        ncols = cols_arr.size
    out = [np.zeros((M, ncols), np.float64) for _ in range(5)]
    rc = _load().ora_swiglu_linear(_ptr(packed), _ptr(scales), float(gs), _ptr(x_bf16), M, N2,
                                   K, _ptr(cols_arr), ncols, *[_ptr(o) for o in out], nthreads)
    if rc:
        raise ValueError("ora_swiglu_linear failed (%d)" % rc)
    return tuple(out)


# sup over v of |d silu / dv| is 1.0998 (at v = 2.3994); rounded up
SILU_LIPSCHITZ = 1.1


def swiglu_tolerance(h_ref, gate, up, absdot_gate, absdot_up) -> np.ndarray:
    """Bound on |h - h_ref| for a kernel whose gate and up values each meet the
    linear's bound and whose output is rounded to bf16: with tg, tu the linear
    bounds of gate and up and L the Lipschitz constant of SiLU,
        |silu(g') u' - silu(g) u| <= L tg (|u| + tu) + |silu(g)| tu,
    plus the bf16 rounding of the result (relative 2^-9, taken as 2^-8)."""
    tg = tolerance(gate, absdot_gate)
    tu = tolerance(up, absdot_up)
    sg = np.abs(np.vectorize(silu, otypes=[np.float64])(gate)) if np.size(gate) else np.abs(gate)
    b = SILU_LIPSCHITZ * tg * (np.abs(up) + tu) + sg * tu
    return (1.0 + 2.0 ** -8) * b + 2.0 ** -8 * np.abs(h_ref)


def topk(y, k: int) -> np.ndarray:
    """Indices [M][k] of the k largest entries of each row of y (fp64 [M][N]),
    largest first, ties by ascending index; k = 1 is the greedy argmax."""
    y = _c(np.atleast_2d(y), np.float64)
    M, N = y.shape
    idx = np.zeros((M, k), np.int64)
    rc = _load().ora_topk(_ptr(y), M, N, k, _ptr(idx))
    if rc:
        raise ValueError("ora_topk failed (%d)" % rc)
    return idx


def argmax_decided(y_ref, tol) -> tuple:
    """(argmax [M], decided [M]): the oracle's greedy choice per row, and
    whether it is decided within tolerance, i.e. the reference top-2 gap
    exceeds the sum of the two logits' bounds (else a kernel may pick the
    runner-up; reading R10)."""
    y_ref = np.atleast_2d(np.asarray(y_ref, np.float64))
    tol = np.atleast_2d(np.asarray(tol, np.float64))
    if y_ref.shape[1] < 2:
        return topk(y_ref, 1)[:, 0], np.ones(y_ref.shape[0], bool)
    t2 = topk(y_ref, 2)
    r = np.arange(y_ref.shape[0])
    a, b = t2[:, 0], t2[:, 1]
    decided = y_ref[r, a] - y_ref[r, b] > tol[r, a] + tol[r, b]
    return a, decided


def quantize_x(x_bf16, gs_x=None, nthreads: int = NTHREADS):
    """NVFP4 activations for the W4A4 tier: X bf16 [M][K] -> (packed [M][K/2],
    scales [M][K/16], gs_x). gs_x is the per-tensor input scale; None takes
    amax(|X|) / (6 * 448) of this X. The steps are the weight quantiser's."""
    x_bf16 = _c(x_bf16, np.uint16)
    x = bf16_bits_to_f64(x_bf16).astype(np.float32)          # exact
    if gs_x is None:
        gs_x = global_scale(x, nthreads)
    packed, scales = quantize_rows(x, float(gs_x), nthreads)
    return packed, scales, float(gs_x)


def _rows_arg(rows, N):
    if rows is None:
        return None, N
    r = _c(rows, np.int64)
    return r, r.size


def linear_w4a4(w_packed, w_scales, gs_w, x_packed, x_scales, gs_x, M, N, K, rows=None,
                nthreads: int = NTHREADS):
    """W4A4 reference linear. Returns (y fp64 [M][nrows], absdot fp64 [M][nrows])."""
    arrs = [_c(a, np.uint8) for a in (w_packed, w_scales, x_packed, x_scales)]
    rows_arr, nrows = _rows_arg(rows, N)
    y = np.zeros((M, nrows), np.float64)
    ad = np.zeros((M, nrows), np.float64)
    rc = _load().ora_linear_w4a4(_ptr(arrs[0]), _ptr(arrs[1]), float(gs_w), _ptr(arrs[2]),
                                 _ptr(arrs[3]), float(gs_x), M, N, K, _ptr(rows_arr), nrows,
                                 _ptr(y), _ptr(ad), nthreads)
    if rc:
        raise ValueError("ora_linear_w4a4 failed (%d)" % rc)
    return y, ad


def quantize_fp8_rows(w, nthreads: int = NTHREADS):
    """FP8 weight tier: w fp32 [N][K] -> (codes uint8 [N][K], row scales fp32 [N])."""
    w = _c(w, np.float32)
    N, K = w.shape
    codes = np.zeros((N, K), np.uint8)
    sc = np.zeros(N, np.float32)
    rc = _load().ora_quantize_fp8_rows(_ptr(w), N, K, _ptr(codes), _ptr(sc), nthreads)
    if rc:
        raise ValueError("ora_quantize_fp8_rows failed (%d)" % rc)
    return codes, sc


def linear_fp8(codes, row_scales, x_bf16, M, N, K, rows=None, nthreads: int = NTHREADS):
    """FP8 weight tier reference linear. Returns (y, absdot), fp64 [M][nrows]."""
    codes = _c(codes, np.uint8)
    row_scales = _c(row_scales, np.float32)
    x_bf16 = _c(x_bf16, np.uint16)
    rows_arr, nrows = _rows_arg(rows, N)
    y = np.zeros((M, nrows), np.float64)
    ad = np.zeros((M, nrows), np.float64)
    rc = _load().ora_linear_fp8(_ptr(codes), _ptr(row_scales), _ptr(x_bf16), M, N, K,
                                _ptr(rows_arr), nrows, _ptr(y), _ptr(ad), nthreads)
    if rc:
        raise ValueError("ora_linear_fp8 failed (%d)" % rc)
    return y, ad


def bf16_round_array(v: np.ndarray) -> np.ndarray:
    """Element-wise ora_bf16_rne over an fp64 array (bit patterns)."""
    f = _load().ora_bf16_rne
    flat = np.asarray(v, np.float64).ravel()
    return np.array([f(float(t)) for t in flat], np.uint16).reshape(np.shape(v))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)
