"""Measure every variant of the NVFP4 linear on a set of (M, N, K) shapes and
write the table that AUTO plans choose from (csrc/variant_table.csv).

    python -m nvfp4_weight_streaming_b200.tune_variants [--out PATH] [--quick]

Each shape is timed per variant as the median of three blocks of back-to-back
calls replayed from a CUDA graph (programmatic dependent launch on), with
byte-identical weight copies rotated so the footprint exceeds four times the
L2 cache: the same method as the benchmark, on random weights quantised on
the device by nvfp4_quantize. A variant that cannot take a shape is left
empty. The library picks, for a plan's (M, N, K), the fastest variant of the
nearest measured shape (csrc/variant_table.inc, generated from the CSV by
gen_variant_table.py when the library is built).
"""
from __future__ import annotations

import argparse
import math
import os
import statistics

HERE = os.path.dirname(os.path.abspath(__file__))
DEFAULT_OUT = os.path.join(HERE, "csrc", "variant_table.csv")

# (M, N, K): the projections the library is built for -- decode and
# speculative verification of a fused gate+up projection (K 5120, N 34816),
# the down projection (K 17408, N 5120), the lm_head (K 5120, N 248320) --
# plus smaller square shapes and the tiny case.
SHAPES = ([(m, 34816, 5120) for m in (1, 2, 4, 8, 12, 16)] +
          [(m, 5120, 17408) for m in (1, 4, 8, 16)] +
          [(m, 248320, 5120) for m in (1, 8, 16)] +
          [(m, 4096, 4096) for m in (1, 4, 16)] +
          [(m, 1024, 1024) for m in (1, 16)] +
          [(1, 512, 256)])
VARIANTS = {"gemv": 1, "mma": 2, "tc": 3, "row": 4}


def time_variant(nv, torch, M, N, K, variant, copies, x, gs, calls=256, repeats=3):
    """Seconds per call, or None if the variant does not take the shape."""
    dev = torch.cuda.current_device()
    try:
        plan = nv.nvfp4_linear_plan(M, N, K, dev, variant | nv.NVFP4_PLAN_PDL)
    except nv.Nvfp4Error as e:
        if e.status == nv.NVFP4_ERR_UNSUPPORTED:
            return None
        raise
    try:
        if nv.nvfp4_linear_variant(plan) != variant:
            return None
        wsb = nv.nvfp4_linear_workspace_bytes(plan)
        ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
        y = torch.empty(M * N, dtype=torch.int16, device="cuda")
        lib = nv.lib()
        stream = torch.cuda.Stream()

        def call(i, h):
            p, s = copies[i % len(copies)]
            st = lib.nvfp4_linear_run(plan, p.data_ptr(), s.data_ptr(), gs.data_ptr(), x.data_ptr(),
                                      y.data_ptr(), ws.data_ptr() if wsb else None, wsb, h)
            if st != 0:
                raise nv.Nvfp4Error(st, "nvfp4_linear_run")

        with torch.cuda.stream(stream):
            for i in range(8):
                call(i, stream.cuda_stream)
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            h = torch.cuda.current_stream().cuda_stream
            for i in range(calls):
                call(i, h)
        with torch.cuda.stream(stream):
            graph.replay()
        stream.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        ts = []
        for _ in range(repeats):
            with torch.cuda.stream(stream):
                e0.record(stream)
                graph.replay()
                e1.record(stream)
            stream.synchronize()
            ts.append(e0.elapsed_time(e1) / 1e3 / calls)
        st = nv.nvfp4_linear_status(plan, ws if wsb else None, stream)
        if st != nv.NVFP4_OK:
            raise nv.Nvfp4Error(st, "device status")
        del graph
        return statistics.median(ts)
    finally:
        nv.nvfp4_linear_destroy(plan)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--out", default=DEFAULT_OUT)
    ap.add_argument("--quick", action="store_true", help="fewer calls per timing block")
    args = ap.parse_args(argv)
    import torch
    import nvfp4_weight_streaming_b200 as nv
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(0)
    rows = []
    for (M, N, K) in SHAPES:
        w = torch.randn((N, K), generator=gen, device="cuda", dtype=torch.float32) * 0.02
        packed = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
        scales = torch.empty((N, K // 16), dtype=torch.uint8, device="cuda")
        gs = torch.empty(1, dtype=torch.float32, device="cuda")
        bad = torch.zeros(1, dtype=torch.int32, device="cuda")
        nv.nvfp4_quantize(w, N, K, packed, scales, gs, bad)
        del w
        wbytes = packed.numel() + scales.numel()
        n = max(1, math.ceil(4.2 * l2 / wbytes))
        copies = [(packed, scales)] + [(packed.clone(), scales.clone()) for _ in range(n - 1)]
        x = (torch.randn((M, K), generator=gen, device="cuda")).to(torch.bfloat16).view(torch.int16)
        times = {}
        for name, v in VARIANTS.items():
            t = time_variant(nv, torch, M, N, K, v, copies, x, gs, calls=64 if args.quick else 256)
            times[name] = t
        best = min((t, name) for name, t in times.items() if t is not None)[1]
        print("M=%-2d N=%-6d K=%-5d %s -> %s" % (M, N, K, "  ".join(
            "%s %.2f" % (k, t * 1e6) if t else "%s -" % k for k, t in times.items()), best), flush=True)
        rows.append((M, N, K, times))
        del copies, packed, scales
        torch.cuda.empty_cache()
    with open(args.out, "w") as f:
        f.write("# Per-call time (us) of each variant of the NVFP4 linear on one B200, written by\n")
        f.write("# python -m nvfp4_weight_streaming_b200.tune_variants; empty: variant not available.\n")
        f.write("M,N,K," + ",".join("%s_us" % k for k in VARIANTS) + "\n")
        for M, N, K, times in rows:
            f.write("%d,%d,%d,%s\n" % (M, N, K, ",".join("%.3f" % (times[k] * 1e6) if times[k] else ""
                                                         for k in VARIANTS)))
    print("wrote", args.out)


if __name__ == "__main__":
    main()
