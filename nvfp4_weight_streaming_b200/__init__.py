"""NVFP4 weight-streaming linear for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in include/nvfp4_linear.h. Every function
here only marshals arguments (device pointers, sizes, a stream handle) into
libnvfp4linear.so; all computation runs in that library's CUDA kernels. There
is no CPU or PyTorch fallback: if the library cannot be built or loaded, the
import fails.

    Y[M][N] = X[M][K] * W^T,  W NVFP4 ([N][K/2] codes, [N][K/16] E4M3 scales,
    one fp32 global scale), X and Y bf16, 1 <= M <= 16.
"""
from __future__ import annotations

import ctypes
import threading

from . import _build

__all__ = [
    "NVFP4_OK", "NVFP4_ERR_INVALID_ARG", "NVFP4_ERR_UNSUPPORTED", "NVFP4_ERR_MISALIGNED",
    "NVFP4_ERR_CUDA", "NVFP4_ERR_TIMEOUT", "NVFP4_ERR_BAD_SCALE", "NVFP4_ERR_WORKSPACE",
    "NVFP4_VARIANT_AUTO", "NVFP4_VARIANT_GEMV", "NVFP4_VARIANT_MMA", "NVFP4_VARIANT_TC",
    "NVFP4_VARIANT_ROW",
    "NVFP4_PLAN_PDL", "NVFP4_PLAN_TEST_STALL", "NVFP4_PLAN_EPI_SWIGLU", "NVFP4_PLAN_EPI_ARGMAX",
    "NVFP4_PLAN_WEIGHT_FP8", "NVFP4_PLAN_ACT_NVFP4", "nvfp4_quantize_fp8",
    "Nvfp4Error", "lib", "library_path",
    "nvfp4_linear_plan", "nvfp4_auto_variant", "nvfp4_linear_workspace_bytes", "nvfp4_linear_variant",
    "nvfp4_linear_split_k", "nvfp4_linear_launches_per_run", "nvfp4_linear_run",
    "nvfp4_linear_run_static",
    "NVFP4_STATIC_SCRATCH_BYTES", "nvfp4_linear_status", "nvfp4_linear_destroy",
    "nvfp4_pack_check", "nvfp4_quantize", "nvfp4_status_string", "EXPORTS",
]

NVFP4_OK = 0
NVFP4_ERR_INVALID_ARG = 1
NVFP4_ERR_UNSUPPORTED = 2
NVFP4_ERR_MISALIGNED = 3
NVFP4_ERR_CUDA = 4
NVFP4_ERR_TIMEOUT = 5
NVFP4_ERR_BAD_SCALE = 6
NVFP4_ERR_WORKSPACE = 7

NVFP4_VARIANT_AUTO = 0
NVFP4_VARIANT_GEMV = 1
NVFP4_VARIANT_MMA = 2
NVFP4_VARIANT_TC = 3
NVFP4_VARIANT_ROW = 4
NVFP4_PLAN_PDL = 0x10000
NVFP4_PLAN_EPI_SWIGLU = 0x100
NVFP4_PLAN_EPI_ARGMAX = 0x200
NVFP4_PLAN_WEIGHT_FP8 = 0x1000
NVFP4_PLAN_ACT_NVFP4 = 0x2000
NVFP4_PLAN_TEST_STALL = 0x40000000
NVFP4_STATIC_SCRATCH_BYTES = 16 << 20

_c = ctypes
_P = _c.c_void_p
# name -> (restype, argtypes); the exported C symbols, in header order.
EXPORTS = {
    "nvfp4_linear_plan": (_c.c_int, [_c.c_int, _c.c_int, _c.c_int, _c.c_int, _c.c_uint,
                                     _c.POINTER(_P)]),
    "nvfp4_auto_variant": (_c.c_int, [_c.c_int, _c.c_int, _c.c_int]),
    "nvfp4_linear_workspace_bytes": (_c.c_size_t, [_P]),
    "nvfp4_linear_variant": (_c.c_int, [_P]),
    "nvfp4_linear_split_k": (_c.c_int, [_P]),
    "nvfp4_linear_launches_per_run": (_c.c_int, [_P]),
    "nvfp4_linear_run": (_c.c_int, [_P, _P, _P, _P, _P, _P, _P, _c.c_size_t, _P]),
    "nvfp4_linear_run_static": (_c.c_int, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "nvfp4_linear_status": (_c.c_int, [_P, _P, _P]),
    "nvfp4_linear_destroy": (None, [_P]),
    "nvfp4_pack_check": (_c.c_int, [_P, _P, _P, _c.c_int, _c.c_int, _P, _P, _P]),
    "nvfp4_quantize": (_c.c_int, [_P, _c.c_int, _c.c_int, _P, _P, _P, _P, _P]),
    "nvfp4_quantize_fp8": (_c.c_int, [_P, _c.c_int, _c.c_int, _P, _P, _P, _P]),
    "nvfp4_status_string": (_c.c_char_p, [_c.c_int]),
}

_lock = threading.Lock()
_lib = None


class Nvfp4Error(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__("%s: %s (status %d)" % (what or "nvfp4", _status_text(status), status))


def library_path() -> str:
    return _build.LIB


def lib():
    """The loaded CUDA library (built in place first if missing or stale)."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            L = ctypes.CDLL(path)
            for name, (res, args) in EXPORTS.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
        return _lib


def _status_text(s: int) -> str:
    try:
        return lib().nvfp4_status_string(s).decode()
    except Exception:  # library not loadable: still report the number
        return "status"


def _check(s: int, what: str) -> int:
    if s != NVFP4_OK:
        raise Nvfp4Error(s, what)
    return s


def _ptr(t) -> int | None:
    """Device pointer of a torch tensor, an int, or None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


# ---- the C ABI, same names ------------------------------------------------

def nvfp4_linear_plan(M: int, N: int, K: int, device: int = 0, flags: int = 0):
    """Returns an opaque plan handle (int). Raises Nvfp4Error on failure."""
    h = _P()
    _check(lib().nvfp4_linear_plan(M, N, K, device, flags, ctypes.byref(h)), "nvfp4_linear_plan")
    return h.value


def nvfp4_linear_workspace_bytes(plan) -> int:
    return int(lib().nvfp4_linear_workspace_bytes(plan))


def nvfp4_linear_variant(plan) -> int:
    return int(lib().nvfp4_linear_variant(plan))


def nvfp4_auto_variant(M: int, N: int, K: int) -> int:
    """Variant an AUTO plan of this shape starts from (host-only query)."""
    return int(lib().nvfp4_auto_variant(M, N, K))


def nvfp4_linear_split_k(plan) -> int:
    return int(lib().nvfp4_linear_split_k(plan))


def nvfp4_linear_launches_per_run(plan) -> int:
    return int(lib().nvfp4_linear_launches_per_run(plan))


def nvfp4_linear_run(plan, w_packed, w_scales, w_global, x, y, workspace=None, ws_bytes=None,
                     stream=None, check: bool = True) -> int:
    """Launch Y = X W^T. Tensors (or raw device pointers) as in the C header."""
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size() if hasattr(workspace, "numel") else 0
    s = lib().nvfp4_linear_run(plan, _ptr(w_packed), _ptr(w_scales), _ptr(w_global), _ptr(x),
                               _ptr(y), _ptr(workspace), ws_bytes, _stream(stream))
    return _check(s, "nvfp4_linear_run") if check else s


def nvfp4_linear_run_static(plan, w_packed, w_scales, w_global, x, y, status_out=None,
                            stream=None, check: bool = True) -> int:
    """Launch Y = X W^T with the split-K scratch in the library's fixed device
    array instead of a caller workspace (nothing is allocated). status_out: an
    optional device uint32 that receives the run's status word."""
    s = lib().nvfp4_linear_run_static(plan, _ptr(w_packed), _ptr(w_scales), _ptr(w_global),
                                      _ptr(x), _ptr(y), _ptr(status_out), _stream(stream))
    return _check(s, "nvfp4_linear_run_static") if check else s


def nvfp4_linear_status(plan, workspace=None, stream=None) -> int:
    return int(lib().nvfp4_linear_status(plan, _ptr(workspace), _stream(stream)))


def nvfp4_linear_destroy(plan) -> None:
    lib().nvfp4_linear_destroy(plan)


def nvfp4_pack_check(w_packed, w_scales, w_global, N: int, K: int, w_bf16_out, d_bad,
                     stream=None, check: bool = True) -> int:
    s = lib().nvfp4_pack_check(_ptr(w_packed), _ptr(w_scales), _ptr(w_global), N, K,
                               _ptr(w_bf16_out), _ptr(d_bad), _stream(stream))
    return _check(s, "nvfp4_pack_check") if check else s


def nvfp4_quantize(w, N: int, K: int, w_packed, w_scales, w_global, d_bad=None, stream=None,
                   check: bool = True) -> int:
    s = lib().nvfp4_quantize(_ptr(w), N, K, _ptr(w_packed), _ptr(w_scales), _ptr(w_global),
                             _ptr(d_bad), _stream(stream))
    return _check(s, "nvfp4_quantize") if check else s


def nvfp4_quantize_fp8(w, N: int, K: int, codes, row_scales, d_bad=None, stream=None,
                       check: bool = True) -> int:
    s = lib().nvfp4_quantize_fp8(_ptr(w), N, K, _ptr(codes), _ptr(row_scales), _ptr(d_bad),
                                 _stream(stream))
    return _check(s, "nvfp4_quantize_fp8") if check else s


def nvfp4_status_string(s: int) -> str:
    return lib().nvfp4_status_string(s).decode()
