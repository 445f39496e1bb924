"""The C-ABI library: it builds, loads, and exports every symbol the header
declares; argument checks that need no device. No compute calls here."""
import ctypes
import os
import re

import pytest

import nvfp4_weight_streaming_b200 as nv
from tests.conftest import ROOT


def header_functions():
    src = open(os.path.join(ROOT, "include", "nvfp4_linear.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    fns = header_functions()
    for name in ("nvfp4_linear_plan", "nvfp4_linear_run", "nvfp4_pack_check",
                 "nvfp4_linear_status", "nvfp4_linear_destroy", "nvfp4_status_string",
                 "nvfp4_linear_workspace_bytes"):
        assert name in fns


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(nv._build.build())
    for name in header_functions():
        assert hasattr(L, name), name
    assert set(header_functions()) == set(nv.EXPORTS)


def test_status_strings():
    for s in range(8):
        assert nv.nvfp4_status_string(s)
    assert nv.nvfp4_status_string(nv.NVFP4_ERR_TIMEOUT) == "device wait timed out"


@pytest.mark.parametrize("M,N,K", [(0, 8, 256), (17, 8, 256), (1, -1, 256), (1, 8, 100),
                                    (1, 8, -256)])
def test_plan_rejects_bad_shapes_before_touching_a_device(M, N, K):
    h = ctypes.c_void_p()
    s = nv.lib().nvfp4_linear_plan(M, N, K, 0, 0, ctypes.byref(h))
    assert s == nv.NVFP4_ERR_INVALID_ARG and h.value is None


def test_null_arguments_rejected():
    L = nv.lib()
    assert L.nvfp4_linear_plan(1, 8, 256, 0, 0, None) == nv.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_linear_run(None, None, None, None, None, None, None, 0, None) == \
        nv.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_linear_status(None, None, None) == nv.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_linear_workspace_bytes(None) == 0
    assert L.nvfp4_linear_variant(None) == -1
    assert L.nvfp4_linear_launches_per_run(None) == -1
    L.nvfp4_linear_destroy(None)
    assert L.nvfp4_pack_check(None, None, None, 4, 17, None, None, None) == \
        nv.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_quantize(None, 4, 16, None, None, None, None, None) == \
        nv.NVFP4_ERR_INVALID_ARG


def test_library_does_not_load_the_oracle():
    # The product library and the oracle share no code: no oracle symbol is
    # reachable from the product library.
    L = ctypes.CDLL(nv._build.build())
    assert not hasattr(L, "ora_linear")
    src_dir = os.path.join(ROOT, "nvfp4_weight_streaming_b200")
    for dirpath, _, files in os.walk(src_dir):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "nvfp4_oracle" not in text, f
