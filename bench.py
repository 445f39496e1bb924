#!/usr/bin/env python
"""Benchmark of the NVFP4 weight-streaming linear on B200.

Metric: effective HBM bandwidth of Y[M,N] = X[M,K] W^T, counting
bytes = N*K/2 + N*K/16 + 2*M*K + 2*M*N per call (packed codes, E4M3 scales,
X and Y), reported in GB/s and as a fraction of the measured device-copy peak.
One "step" is one call of the linear on one batch of M tokens. The headline
workload is the single-token decode projection M=1, K=5120, N=34816 (a fused
gate+up of a 27B-class decoder with hidden size 5120).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torch.distributed.run) every rank runs its own replica
of the workload (replicas only: the linear needs no exchange); the time is the
maximum over ranks and the value the bytes of all ranks over that time.
Inputs are synthetic (seeded generators in synth/), weights rotate over enough
byte-identical copies that the footprint is > 4x the L2 cache.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# calls per timed block of a sweep point (the headline uses --steps): a few
# seconds of timed work even for the 715 MB lm_head
SWEEP_CALLS = 2000
METRIC = "NVFP4 linear effective HBM GB/s and % of peak at M=1/16 (27B-class shapes)"
NOMINAL_HBM_GBS = 8000.0
VARIANT_NAMES = ("auto", "gemv", "mma", "tc", "row")
FALLBACK_HBM_GBS = 6650.0


def bytes_per_call(M: int, N: int, K: int, fmt: str = "nvfp4", epi: str = "none") -> int:
    """Algorithmic bytes of one call: weights (NVFP4 codes and E4M3 scales, or
    FP8 codes and fp32 row scales), X (bf16; the W4A4 tier quantises it in the
    kernel), and the output (Y; N/2 columns with the SwiGLU epilogue; an int32
    index and a float value per token with argmax)."""
    wbytes = N * K // 2 + N * K // 16 if fmt in ("nvfp4", "w4a4") else N * K + 4 * N
    out = {"none": 2 * M * N, "swiglu": M * N, "argmax": 8 * M}[epi]
    return wbytes + 2 * M * K + out


def effective_gbs(nbytes: float, seconds: float) -> float:
    return nbytes / seconds / 1e9


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled while work runs."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, period_ms: int = 50):
        self.index = index
        self.period_ms = period_ms
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", str(self.period_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        return self.summarize(out)

    def summarize(self, out: str):
        """Median SM clock, max clock and the throttle reasons seen Active in
        the samples inside the timed region [t0, t1] (60 ms margin)."""
        import datetime
        rows = [r.split(",") for r in out.strip().splitlines() if r.strip()]
        sm, smax, reasons, total = [], None, set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [c.strip() for c in r]
            try:
                ts = datetime.datetime.strptime(r[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                mhz, mx = float(r[2]), float(r[3])
            except (ValueError, IndexError):
                continue
            total += 1
            # keep the samples taken inside the timed region (small margin)
            if self.t0 is not None and not (self.t0 - 0.06 <= ts <= self.t1 + 0.06):
                continue
            sm.append(mhz)
            smax = mx
            for name, val in zip(names, r[6:10]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm), "samples_total": total}


def dist_setup(n_gpus: int):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        if torch.cuda.is_available():
            torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _reduce(world, value: float, op) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    device = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(world, value: float) -> float:
    """Timing across replicas: the slowest rank defines the step time."""
    import torch.distributed as dist
    return _reduce(world, value, dist.ReduceOp.MAX if world > 1 else None)


def sum_over_ranks(world, value: float) -> float:
    import torch.distributed as dist
    return _reduce(world, value, dist.ReduceOp.SUM if world > 1 else None)


def aggregate(world: int, bytes_per_call: float, sec_per_call_this_rank: float):
    """(seconds per call = max over ranks, whole-job GB/s = all ranks' bytes / that time)."""
    sec = max_over_ranks(world, sec_per_call_this_rank)
    total_bytes = sum_over_ranks(world, bytes_per_call)
    return sec, effective_gbs(total_bytes, sec)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

class Problem:
    """One workload on the device: weight copies, X, Y, plan, workspace.
    fmt "nvfp4" (the method), "w4a4" (NVFP4 weights, X quantised to NVFP4 in the
    kernel) or "fp8" (the comparison tier); epi "none",
    "swiglu" or "argmax" (fused epilogues)."""

    def __init__(self, name: str, M: int, variant: int, min_footprint: float, flags: int = 0,
                 fmt: str = "nvfp4", epi: str = "none"):
        import numpy as np
        import torch
        import synth
        import nvfp4_weight_streaming_b200 as nv
        self.nv = nv
        wl = synth.WORKLOADS[name]
        self.name, self.M, self.N, self.K = name, M, wl.N, wl.K
        dev = torch.cuda.current_device()
        self.fmt, self.epi = fmt, epi
        # weights: generated on the host, quantised on the device by the library
        W = torch.from_numpy(synth.weights_f32(wl)).cuda()
        bad = torch.zeros(1, dtype=torch.int32, device="cuda")
        if fmt in ("nvfp4", "w4a4"):
            if fmt == "w4a4":
                flags |= nv.NVFP4_PLAN_ACT_NVFP4
            packed = torch.empty((self.N, self.K // 2), dtype=torch.uint8, device="cuda")
            scales = torch.empty((self.N, self.K // 16), dtype=torch.uint8, device="cuda")
            gs = torch.empty(1, dtype=torch.float32, device="cuda")
            nv.nvfp4_quantize(W, self.N, self.K, packed, scales, gs, bad)
        else:
            packed = torch.empty((self.N, self.K), dtype=torch.uint8, device="cuda")
            scales = torch.empty(self.N, dtype=torch.float32, device="cuda")
            gs = torch.ones(1, dtype=torch.float32, device="cuda")
            nv.nvfp4_quantize_fp8(W, self.N, self.K, packed, scales, bad)
            flags |= nv.NVFP4_PLAN_WEIGHT_FP8
        flags |= {"none": 0, "swiglu": nv.NVFP4_PLAN_EPI_SWIGLU, "argmax": nv.NVFP4_PLAN_EPI_ARGMAX}[epi]
        torch.cuda.synchronize()
        assert int(bad.item()) == 0
        del W
        wbytes = packed.numel() * packed.element_size() + scales.numel() * scales.element_size()
        self.ncopies = max(1, math.ceil(min_footprint / wbytes))
        self.copies = [(packed, scales)] + [(packed.clone(), scales.clone())
                                            for _ in range(self.ncopies - 1)]
        self.gs = gs
        xh = synth.x_bf16(wl, M)
        self.x_host = xh
        self.x = torch.from_numpy(xh.view(np.int16)).cuda()
        ycount = {"none": M * self.N, "swiglu": M * (self.N // 2), "argmax": 4 * M}[epi]
        self.y = torch.empty(ycount, dtype=torch.int16, device="cuda")
        self.plan = nv.nvfp4_linear_plan(M, self.N, self.K, dev, variant | flags)
        self.flags = flags
        self.variant = nv.nvfp4_linear_variant(self.plan)
        self.split_k = nv.nvfp4_linear_split_k(self.plan)
        self.wsb = nv.nvfp4_linear_workspace_bytes(self.plan)
        self.ws = torch.zeros(max(self.wsb, 16), dtype=torch.uint8, device="cuda")
        self.bytes = bytes_per_call(M, self.N, self.K, fmt, epi)
        self.footprint = wbytes * self.ncopies
        self.lib = nv.lib()

    def call(self, i: int, stream_handle: int):
        p, s = self.copies[i % self.ncopies]
        st = self.lib.nvfp4_linear_run(self.plan, p.data_ptr(), s.data_ptr(), self.gs.data_ptr(),
                                       self.x.data_ptr(), self.y.data_ptr(),
                                       self.ws.data_ptr() if self.wsb else None, self.wsb,
                                       stream_handle)
        if st != 0:
            raise RuntimeError("nvfp4_linear_run failed: %s" % self.nv.nvfp4_status_string(st))

    def check_status(self):
        import torch
        st = self.nv.nvfp4_linear_status(self.plan, self.ws if self.wsb else None,
                                         torch.cuda.current_stream())
        if st != 0:
            raise RuntimeError("device status: %s" % self.nv.nvfp4_status_string(st))

    def destroy(self):
        self.nv.nvfp4_linear_destroy(self.plan)


def time_problem(pb: Problem, steps: int, warmup: int, world: int, graph_len: int = 64,
                 sampler: ClockSampler | None = None, repeats: int = 1):
    """Warm up, then time exactly `steps` calls (replayed from CUDA graphs of
    `graph_len` calls) between CUDA events, `repeats` times; returns the
    median seconds per call (each repeat's time is the max over ranks), the
    number of kernel launches in one timed block, and every repeat's seconds
    per call."""
    import torch
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        h = stream.cuda_stream
        for i in range(max(3, warmup)):
            pb.call(i, h)
    stream.synchronize()
    pb.check_status()
    glen = max(1, min(graph_len, steps))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        h = torch.cuda.current_stream().cuda_stream
        for i in range(glen):
            pb.call(i, h)
    tail = steps % glen
    tail_graph = None
    if tail:
        tail_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(tail_graph, stream=stream):
            h = torch.cuda.current_stream().cuda_stream
            for i in range(tail):
                pb.call(i, h)
    # untimed replay so the graphs are uploaded and warm
    with torch.cuda.stream(stream):
        graph.replay()
    stream.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    per_call = []
    for rep in range(max(1, repeats)):
        barrier(world)
        torch.cuda.synchronize()
        if sampler and rep == 0:
            sampler.mark("t0")
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(steps // glen):
                graph.replay()
            if tail_graph is not None:
                tail_graph.replay()
            e1.record(stream)
        stream.synchronize()
        torch.cuda.synchronize()
        barrier(world)
        per_call.append(max_over_ranks(world, e0.elapsed_time(e1) / 1e3) / steps)
    if sampler:
        sampler.mark("t1")
    pb.check_status()
    del graph, tail_graph
    return (statistics.median(per_call), steps * pb.nv.nvfp4_linear_launches_per_run(pb.plan),
            per_call)


def time_e2e(pb: Problem, steps: int, world: int):
    """Same metric through the public API with host buffers: each step copies
    the weight copy and X from pinned host memory, runs, reads Y back."""
    import numpy as np
    import torch
    p, s = pb.copies[0]
    hp = torch.empty(p.shape, dtype=torch.uint8).pin_memory()
    hs = torch.empty(s.shape, dtype=torch.uint8).pin_memory()
    hp.copy_(p.cpu())
    hs.copy_(s.cpu())
    hx = torch.from_numpy(pb.x_host.view(np.int16)).pin_memory()
    hy = torch.empty(pb.y.shape, dtype=torch.int16).pin_memory()
    stream = torch.cuda.current_stream()
    h = stream.cuda_stream

    def step():
        p.copy_(hp, non_blocking=True)
        s.copy_(hs, non_blocking=True)
        pb.x.copy_(hx, non_blocking=True)
        pb.call(0, h)
        hy.copy_(pb.y, non_blocking=True)

    for _ in range(2):
        step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    sec = max_over_ranks(world, e0.elapsed_time(e1) / 1e3) / steps
    h2d = hp.numel() + hs.numel() + hx.numel() * 2
    d2h = hy.numel() * 2
    return sec, h2d, d2h


def cpu_baseline(sample_rows: int = 34816, M: int = 1):
    """The oracle, as it stands, on the host cores: quantise the decode
    workload's weights (oracle quantiser) and time its fp64 linear on
    `sample_rows` rows."""
    import numpy as np
    import oracle
    import synth
    wl = synth.WORKLOADS["decode"]
    rows = min(sample_rows, wl.N)
    W = synth.weights_f32(wl, rows=slice(0, rows))
    gs = oracle.global_scale(synth.weights_f32(wl))
    packed, scales = oracle.quantize_rows(W, gs)
    X = synth.x_bf16(wl, M)
    cores = oracle.threads_for(rows, oracle.NTHREADS)    # threads the oracle uses here
    oracle.linear(packed, scales, gs, X, M, rows, wl.K, nthreads=oracle.NTHREADS)   # warm-up
    ts = []
    for _ in range(3):
        t0 = time.perf_counter()
        oracle.linear(packed, scales, gs, X, M, rows, wl.K, nthreads=oracle.NTHREADS)
        ts.append(time.perf_counter() - t0)
    t = statistics.median(ts)
    return {"value": effective_gbs(bytes_per_call(M, rows, wl.K), t), "unit": "GB/s",
            "cores": cores, "kind": "oracle",
            "sample": "fp64 oracle linear, decode workload M=%d K=%d, first %d of %d rows, "
                      "median of 3" % (M, wl.K, rows, wl.N)}


def measured_traffic(variant: str, workload: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    record (profiles/traffic.json), or None when the kernel's sources have
    changed since the capture or the capture was of another workload."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    kernel = {"mma": "k_mma", "w4a4-tc": "k_tc4"}.get(variant)
    if kernel is None or not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(kernel)
    if not rec or rec.get("workload") != workload:
        return None
    if sources_digest(rec["sources"]) != rec["sources_sha256"]:
        return None
    return rec["traffic_bytes_per_launch"]


def sources_digest(paths) -> str:
    """sha256 of the C++/CUDA sources with comments and whitespace removed, so
    that editing a comment does not count as changing the kernel."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in paths:
        text = open(os.path.join(ROOT, f)).read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()


def run_ours(args):
    import torch
    world, rank, local = dist_setup(args.gpus)
    import nvfp4_weight_streaming_b200 as nv
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20)
    peak, peak_kind = peaks()
    variant = {"auto": 0, "gemv": 1, "mma": 2, "tc": 3, "row": 4}[args.variant]
    flags = 0 if args.no_pdl else nv.NVFP4_PLAN_PDL
    pb = Problem(args.workload, args.M, variant, min_footprint=4.2 * l2, flags=flags, fmt=args.fmt)
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if sampler:
        sampler.start()
    sec, launches, reps = time_problem(pb, args.steps, args.warmup, world, sampler=sampler,
                                       repeats=args.repeats)
    clocks = sampler.stop() if sampler else None
    value = effective_gbs(pb.bytes * world, sec)
    per_gpu = effective_gbs(pb.bytes, sec)
    sweep = []
    if not args.no_sweep and world == 1:
        # every workload shape and M (the down projection's 64 rotated copies
        # included), then the fused epilogues and the FP8 comparison tier;
        # single-GPU runs only, SWEEP_CALLS calls per timed block
        points = [("verify", m, "nvfp4", "none") for m in (1, 2, 4, 8, 12, 16)] + \
                 [("down", m, "nvfp4", "none") for m in (1, 4, 8, 16)] + \
                 [("lm_head", m, "nvfp4", "none") for m in (1, 8, 16)] + \
                 [("verify", m, "nvfp4", "swiglu") for m in (1, 16)] + \
                 [("lm_head", m, "nvfp4", "argmax") for m in (1, 16)] + \
                 [("verify", m, "fp8", "none") for m in (1, 2, 16)] + \
                 [("down", 1, "fp8", "none"), ("lm_head", 1, "fp8", "none")]
        points = [pt + (None,) for pt in points]
        # W4A4 on both of its variants: decoded for the warp MMA, and the
        # block-scaled FP4 tensor cores
        for v4 in (nv.NVFP4_VARIANT_MMA, nv.NVFP4_VARIANT_TC):
            points += [("verify", m, "w4a4", "none", v4) for m in (1, 4, 16)] + \
                      [("down", m, "w4a4", "none", v4) for m in (1, 16)]
        points += [("lm_head", 1, "w4a4", "none", nv.NVFP4_VARIANT_TC)]
        base_us = {}
        for (name, M, fmt, epi, forced) in points:
            v = forced if forced is not None else variant if (fmt == "nvfp4" and epi == "none") else 0
            q = Problem(name, M, v, min_footprint=4.2 * l2, flags=flags, fmt=fmt, epi=epi)
            s2, _, r2 = time_problem(q, max(min(args.steps, SWEEP_CALLS), 200), args.warmup, world,
                                     repeats=args.repeats)
            g = effective_gbs(q.bytes, s2)
            pt = {"workload": name, "M": M, "N": q.N, "K": q.K,
                  "weights": "nvfp4" if fmt == "w4a4" else fmt,
                  "activations": "nvfp4 (quantised in the kernel)" if fmt == "w4a4" else "bf16",
                  "epilogue": epi,
                  "variant": VARIANT_NAMES[q.variant], "split_k": q.split_k,
                  "bytes_per_call": q.bytes, "us_per_call": s2 * 1e6,
                  "us_spread": [min(r2) * 1e6, max(r2) * 1e6], "GBps": g,
                  "frac_of_measured_peak": g / peak}
            if fmt == "nvfp4" and epi == "none":
                base_us[(name, M)] = s2 * 1e6
            elif (name, M) in base_us:
                pt["time_over_plain_nvfp4"] = s2 * 1e6 / base_us[(name, M)]
            sweep.append(pt)
            q.destroy()
            del q
            torch.cuda.empty_cache()
    e2e = None
    if not args.no_e2e:
        esec, h2d, d2h = time_e2e(pb, max(3, min(args.steps, 20)), world)
        e2e = {"value": effective_gbs(pb.bytes * world, esec), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
            "repeats": len(reps), "ms_per_step_spread": [min(reps) * 1e3, max(reps) * 1e3],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": {"nvfp4": "nvfp4 weights x bf16 activations, f16 products, f32 accumulate",
                      "w4a4": "nvfp4 weights x nvfp4 activations (quantised on the device), "
                              "f32 accumulate",
                      "fp8": "e4m3 weights x bf16 activations, f16 products, f32 accumulate"}[args.fmt],
            "data": "synthetic (seeded SplitMix64/Box-Muller, workload recipes in synth/)",
            "config": {"workload": "%s projection M=%d K=%d N=%d" % (args.workload, pb.M, pb.K, pb.N),
                       "M": pb.M, "K": pb.K, "N": pb.N, "tier": args.fmt,
                       "variant": VARIANT_NAMES[pb.variant],
                       "split_k": pb.split_k, "bytes_per_call": pb.bytes,
                       "l2": "inputs larger than L2: %d byte-identical weight copies "
                             "rotated, %.0f MB > %.1f x %.0f MB L2" %
                             (pb.ncopies, pb.footprint / 1e6, pb.footprint / l2, l2 / 1e6),
                       "launch": "CUDA graphs of back-to-back calls on one stream" +
                                 ("" if args.no_pdl else
                                  ", programmatic dependent launch (a call streams its weights "
                                  "while the previous call finishes)"),
                       "parallelism": "replicas x%d" % world},
            "pct_of_measured_peak": 100 * per_gpu / peak,
            "pct_of_nominal_8TBps": 100 * per_gpu / NOMINAL_HBM_GBS,
            "roofline": {"bound": "hbm", "achieved": per_gpu, "peak": peak, "unit": "GB/s",
                         "frac": per_gpu / peak,
                         "traffic": measured_traffic(VARIANT_NAMES[pb.variant] if args.fmt == "nvfp4"
                                                     else args.fmt + "-" + VARIANT_NAMES[pb.variant],
                                                     "%s projection M=%d K=%d N=%d" %
                                                     (args.workload, pb.M, pb.K, pb.N)),
                         "peak_kind": peak_kind + " device-copy bandwidth (MEASURED_PEAKS hbm_gbs)"},
            "gpu_launches": launches,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "sweep": sweep,
        }
        print(json.dumps(line), flush=True)
    pb.destroy()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# reference arm: the oracle on the host cores
# ---------------------------------------------------------------------------

def run_reference(args):
    """The oracle as it stands, timed on the host cores over `steps` calls
    after `warmup` calls, each call on a row sample of the workload. The
    sample is sized so that the whole run takes about --reference-budget
    seconds (unless --reference-rows fixes it); `cores` reports the threads
    the oracle actually used for that sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    import synth
    wl = synth.WORKLOADS[args.workload]
    M = args.M
    X = synth.x_bf16(wl, M)
    gs = oracle.global_scale(synth.weights_f32(wl))
    calls = max(1, args.steps) + max(0, args.warmup)
    if args.reference_rows:
        rows = max(1, min(wl.N, int(args.reference_rows)))
    else:
        # untimed calibration: seconds per row on one thread
        cal = 256
        p, s = oracle.quantize_rows(synth.weights_f32(wl, rows=slice(0, cal)), gs)
        t0 = time.perf_counter()
        oracle.linear(p, s, gs, X, M, cal, wl.K, nthreads=1)
        per_row = (time.perf_counter() - t0) / cal
        per_call = args.reference_budget / calls
        par_min = next(n for n in (2 ** i for i in range(40)) if oracle.threads_for(n) > 1) \
            if oracle.NTHREADS > 1 else None
        par_rows = int(per_call * oracle.NTHREADS / per_row)
        if par_min is not None and par_rows >= par_min:
            rows = min(wl.N, par_rows)                   # large enough to use every core
        else:
            rows = min(wl.N, (par_min or wl.N + 1) - 1, max(16, int(per_call / per_row)))
    cores = oracle.threads_for(rows)
    packed, scales = oracle.quantize_rows(synth.weights_f32(wl, rows=slice(0, rows)), gs)
    for _ in range(max(0, args.warmup)):
        oracle.linear(packed, scales, gs, X, M, rows, wl.K)
    t0 = time.perf_counter()
    for _ in range(max(1, args.steps)):
        oracle.linear(packed, scales, gs, X, M, rows, wl.K)
    sec = (time.perf_counter() - t0) / max(1, args.steps)
    value = effective_gbs(bytes_per_call(M, rows, wl.K), sec)
    sample = ("each step: fp64 oracle linear on the first %d of %d rows of the %s workload "
              "(M=%d, K=%d) on %d host thread(s), bytes scaled to the sample"
              % (rows, wl.N, args.workload, M, wl.K, cores))
    line = {
        # n_gpus is the launch's world size; the oracle itself runs on rank 0's host cores only
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": max(1, args.steps), "warmup": args.warmup, "ms_per_step": sec * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "%s projection M=%d K=%d N=%d" % (args.workload, M, wl.K, wl.N),
                   "M": M, "K": wl.K, "N": wl.N},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode")
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--variant", choices=list(VARIANT_NAMES), default="auto")
    ap.add_argument("--fmt", choices=["nvfp4", "w4a4", "fp8"], default="nvfp4",
                    help="main problem's tier: NVFP4 weights with bf16 X (the method), X also "
                         "quantised to NVFP4, or FP8 weights")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-pdl", action="store_true",
                    help="launch without programmatic dependent launch")
    ap.add_argument("--repeats", type=int, default=5,
                    help="timed blocks of --steps calls; the median is reported")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--reference-rows", type=int, default=0,
                    help="rows of the workload per reference call (0: sized from the budget)")
    ap.add_argument("--reference-budget", type=float, default=90.0,
                    help="seconds the reference arm's warm-up and timed calls should take")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
