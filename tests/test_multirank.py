"""Replicas on several ranks (CPU, gloo, world size 2): the benchmark's
max-over-ranks timing and whole-job aggregation, and the same collective
sequence on every rank."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        import bench
        # rank 1 is slower: the job's step time is the slowest rank's
        sec_this = 0.002 if rank == 0 else 0.003
        sec, gbs = bench.aggregate(world, 100e6, sec_this)
        bench.barrier(world)
        out[rank] = (sec, gbs)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_replicas_aggregate_with_max_time():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    port = _free_port()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        sec, gbs = out[r]
        assert sec == pytest.approx(0.003)
        assert gbs == pytest.approx(2 * 100e6 / 0.003 / 1e9)


def test_single_rank_aggregate_is_identity():
    import bench
    sec, gbs = bench.aggregate(1, 100e6, 0.002)
    assert sec == 0.002 and gbs == pytest.approx(50.0)


def test_effective_bandwidth_matches_page_read_rate():
    """The metric's arithmetic reproduces the read rate printed on the model
    card (18.80 GiB per token at 81.6 tokens/s -> 1.65 TB/s, ~92% of 1.79)."""
    import bench
    from tests.conftest import read_golden
    d = {k: float(v) for k, v in read_golden("read_rate.txt")}
    gbs = bench.effective_gbs(d["gib_per_token"] * 2 ** 30, 1.0 / d["tokens_per_s"])
    assert round(gbs / 1000, 2) == d["tb_per_s"]
    assert round(100 * gbs / 1000 / d["spec_tb_per_s"]) == d["percent_of_peak"]


def test_bytes_per_call_matches_oracle_model():
    import bench
    import oracle
    for M, N, K in [(1, 34816, 5120), (16, 34816, 5120), (4, 5120, 17408), (8, 248320, 5120)]:
        assert bench.bytes_per_call(M, N, K) == oracle.bytes_model(M, N, K)


def test_bench_traffic_record_matches_current_kernel_sources():
    """The roofline traffic comes from a committed ncu record that is only
    used while the kernel's sources are unchanged."""
    import bench
    t = bench.measured_traffic("mma", "decode projection M=1 K=5120 N=34816")
    assert t is None or 100e6 < t < 120e6
    assert bench.measured_traffic("mma", "some other workload") is None
    assert bench.measured_traffic("tc", "decode projection M=1 K=5120 N=34816") is None


def _bnd_in(lo, hi, L, W):
    """Transcription of the kernels' closed form (unsigned 32-bit steps): the
    number of CTA range boundaries floor(c * L / W), 1 <= c < W, in (lo, hi]."""
    if hi <= lo:
        return 0
    u = 0xFFFFFFFF
    cmin = ((((lo + 1) * W) & u) + L - 1) // L
    cmax = ((((hi + 1) * W) & u) + L - 1) // L - 1
    cmin = max(cmin, 1)
    cmax = min(cmax, W - 1)
    return cmax - cmin + 1 if cmax >= cmin else 0


def test_piece_ordinal_closed_form_matches_enumeration():
    """Stream-K bookkeeping: the ordinal of a piece of a split tile and the
    number of pieces of a tile, as the kernels compute them, equal a direct
    enumeration of the CTA ranges [c*L/W, (c+1)*L/W)."""
    import random
    rnd = random.Random(0)
    cases = [(136 * 20, 148), (20 * 68, 148), (20 * 23, 49), (970 * 20, 148), (4 * 32, 128)]
    cases += [(rnd.randint(1, 4000), rnd.randint(1, 160)) for _ in range(300)]
    for L, W in cases:
        if W > L:
            W = L
        bounds = sorted({c * L // W for c in range(1, W)})
        for _ in range(40):
            lo = rnd.randint(-1, L - 1)
            hi = rnd.randint(lo, L - 1)
            expect = sum(1 for bnd in bounds if lo < bnd <= hi)
            assert _bnd_in(lo, hi, L, W) == expect, (L, W, lo, hi)
        # every tile's piece count for a tile length `cnt` dividing L
        for cnt in (c for c in (5, 20, 23, 68) if L % c == 0):
            for t in range(L // cnt):
                pieces = 1 + sum(1 for b in bounds if t * cnt < b <= (t + 1) * cnt - 1)
                assert 1 + _bnd_in(t * cnt, (t + 1) * cnt - 1, L, W) == pieces


def test_piece_arithmetic_fits_32_bits_for_the_workloads():
    """configure() refuses plans where (units + 1) * P overflows 31 bits; the
    benchmark shapes are far from that."""
    for tiles, steps in ((136, 20), (20, 68), (970, 20), (136, 5)):
        assert (tiles * (steps + 1) + 1) * 148 < 2 ** 31


def test_reference_arm_prints_the_contract_line():
    """bench.py --impl reference (the oracle on the host cores) prints one JSON
    line with the fields the contract asks of the reference arm."""
    import json
    import subprocess
    import sys
    from tests.conftest import ROOT
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                          "--warmup", "1", "--reference-rows", "256"], cwd=ROOT,
                         capture_output=True, text=True, timeout=600, check=True).stdout
    lines = [l for l in out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert "workload" in d["config"]


def test_clock_sampler_keeps_timed_region_and_active_reasons():
    """Host logic of the clocks record: only samples inside the timed region
    count, and a throttle reason is reported when any of them shows it Active."""
    import datetime
    import bench
    t0 = datetime.datetime(2026, 1, 1, 12, 0, 0).timestamp()

    def row(dt, mhz, reasons=("Not Active",) * 4):
        ts = datetime.datetime.fromtimestamp(t0 + dt).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return ", ".join([ts, "0", str(mhz), "1965", "900.5", "0x0"] + list(reasons))

    out = "\n".join([
        row(-1.0, 600, ("Active", "Not Active", "Not Active", "Not Active")),  # before: ignored
        row(0.1, 1800),
        row(0.2, 1900, ("Not Active", "Not Active", "Not Active", "Active")),
        row(0.3, 1950),
        "garbage line",
        row(5.0, 300, ("Not Active", "Active", "Not Active", "Not Active")),   # after: ignored
    ])
    cs = bench.ClockSampler(0)
    cs.t0, cs.t1 = t0, t0 + 0.5
    d = cs.summarize(out)
    assert d["sm_mhz"] == 1900 and d["sm_max_mhz"] == 1965
    assert d["reasons"] == ["sw_power_cap"]
    assert d["samples"] == 3 and d["samples_total"] == 5


def test_reference_arm_under_torchrun_prints_once():
    """Two ranks launched by torchrun: rank 0 alone runs the oracle and prints
    one line, the other rank exits 0 without work."""
    import json
    import socket
    import subprocess
    import sys
    from tests.conftest import ROOT
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                        "--nproc-per-node", "2", "--master-addr", "127.0.0.1", "--master-port",
                        str(port), "bench.py", "--gpus", "2", "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--reference-rows", "128"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1 and lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2


def test_oracle_thread_count_helper():
    """Documented values: one thread below 4096 rows, else the non-empty
    contiguous pieces of the split, never more than asked for."""
    import oracle
    assert oracle.threads_for(0, 8) == 1 and oracle.threads_for(4095, 64) == 1
    assert oracle.threads_for(10 ** 6, 1) == 1
    for n in (4096, 4097, 5000, 34816, 248320):
        for t in (2, 3, 8, 16, 64):
            k = oracle.threads_for(n, t)
            per = -(-n // t)
            assert 1 < k <= t and (k - 1) * per < n <= k * per


def test_reference_arm_sizes_its_sample_to_the_budget():
    """With no fixed row count the reference arm sizes each call from the time
    budget and reports the threads the oracle used for that sample."""
    import json
    import re
    import subprocess
    import sys
    import time
    import oracle
    from tests.conftest import ROOT
    t0 = time.time()
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "300",
                          "--warmup", "3", "--reference-budget", "3"], cwd=ROOT,
                         capture_output=True, text=True, timeout=600, check=True).stdout
    wall = time.time() - t0
    d = json.loads([l for l in out.splitlines() if l.startswith("{")][0])
    rows = int(re.search(r"first (\d+) of", d["cpu_baseline"]["sample"]).group(1))
    assert d["cpu_baseline"]["cores"] == oracle.threads_for(rows)
    assert d["steps"] == 300 and d["ms_per_step"] * 303 < 3 * 1000 * 3   # within 3x the budget
    assert wall < 120
