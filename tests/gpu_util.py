"""Helpers for the GPU parity tests: move host arrays to the device, run the
C-ABI through the binding with guard bytes around every output, compare with
the oracle under the stated tolerance."""
from __future__ import annotations

import numpy as np
import torch

import nvfp4_weight_streaming_b200 as nv
import oracle

GUARD = 64          # elements of guard on each side (multiple of 8: keeps 16 B alignment)
CANARY = 0x5A5A


def dev(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


def host_u16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


class Guarded:
    """A device buffer of `count` int16 elements with canary guards around it."""

    def __init__(self, count: int, dtype=torch.int16, fill=CANARY):
        self.count = count
        self.buf = torch.full((count + 2 * GUARD,), fill if dtype == torch.int16 else 0,
                              dtype=dtype, device="cuda")
        self.view = self.buf[GUARD:GUARD + count]

    def guards_intact(self) -> bool:
        g = torch.cat([self.buf[:GUARD], self.buf[GUARD + self.count:]])
        return bool((g == CANARY).all())


class Weights:
    """An NVFP4 weight set on the device (from host arrays made by the oracle)."""

    def __init__(self, packed: np.ndarray, scales: np.ndarray, gs: float):
        self.N, self.K = packed.shape[0], packed.shape[1] * 2
        self.packed_h, self.scales_h, self.gs = packed, scales, gs
        self.packed = dev(packed)
        self.scales = dev(scales)
        self.gsd = torch.tensor([gs], dtype=torch.float32, device="cuda")


def run_linear(w: Weights, X: np.ndarray, flags: int = 0, plan=None, repeat: int = 1):
    """Run Y = X W^T through the C ABI; returns (y bits [M][N], guards_ok, plan info)."""
    M = X.shape[0]
    own = plan is None
    if own:
        plan = nv.nvfp4_linear_plan(M, w.N, w.K, torch.cuda.current_device(), flags)
    try:
        wsb = nv.nvfp4_linear_workspace_bytes(plan)
        ws = Guarded(max(wsb // 2, 0) + (wsb % 2), fill=0) if wsb else None
        if ws is not None:
            ws.buf[:GUARD] = CANARY
            ws.buf[GUARD + ws.count:] = CANARY
        xd = dev(X)
        y = Guarded(M * w.N)
        stream = torch.cuda.current_stream()
        for _ in range(repeat):
            nv.nvfp4_linear_run(plan, w.packed, w.scales, w.gsd, xd, y.view,
                                None if ws is None else ws.view, wsb, stream)
        st = nv.nvfp4_linear_status(plan, None if ws is None else ws.view, stream)
        assert st == nv.NVFP4_OK, nv.nvfp4_status_string(st)
        ok = y.guards_intact() and (ws is None or ws.guards_intact())
        if ws is not None:
            assert int(ws.view[:2].abs().sum()) == 0, "status word not left zero"
        info = (nv.nvfp4_linear_variant(plan), nv.nvfp4_linear_split_k(plan), wsb)
        return host_u16(y.view).reshape(M, w.N), ok, info
    finally:
        if own:
            nv.nvfp4_linear_destroy(plan)


def check_tolerance(y_bits: np.ndarray, y_ref: np.ndarray, absdot: np.ndarray):
    """Assert |y - y_ref| <= 1e-2 |y_ref| + 1e-4 sum|w x| element by element."""
    y = oracle.bf16_bits_to_f64(y_bits)
    err = np.abs(y - y_ref)
    tol = oracle.tolerance(y_ref, absdot)
    bad = ~(err <= tol)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        details = [(tuple(i), float(y[tuple(i)]), float(y_ref[tuple(i)]), float(tol[tuple(i)]))
                   for i in idx]
        raise AssertionError("%d elements out of tolerance, first: %s" % (bad.sum(), details))
    return float((err / np.maximum(tol, 1e-300)).max())
