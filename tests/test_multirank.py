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
