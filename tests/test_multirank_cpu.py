"""The N > 1 path of bench.py on CPU: two gloo ranks, each timing its own replica; the job time is
the max over ranks and the job throughput counts every rank's units.  (Decode shards by sequence
with no data exchange, so replicas need no collective beyond this reduction.)"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        mine = [1.0 + rank, 5.0 - rank, 2.5]
        got = bench.reduce_max_over_ranks(mine, world)
        q.put((rank, got, bench.job_throughput(1e9, world, got[0])))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict()
    for _ in range(2):
        rank, got, thr = q.get(timeout=120)
        res[rank] = (got, thr)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(2):
        got, thr = res[rank]
        assert got == [2.0, 5.0, 2.5]                 # slowest rank per entry
        assert thr == pytest.approx(2 * 1e9 / 2.0e-3 / 1e9)   # both ranks' bytes over the max time


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_max_over_ranks([3.0, 4.0], 1) == [3.0, 4.0]
    assert bench.job_throughput(2e9, 1, 1.0) == pytest.approx(2000.0)


def test_recorded_traffic_follows_kernel_sources(monkeypatch):
    """A traffic figure is reported only while the kernel sources match the digest it was
    recorded with."""
    import bench
    digest = bench.traffic_sources_digest()
    monkeypatch.setattr(bench, "MEASURED_TRAFFIC", {"w": {"bytes": 123, "sha256": digest, "profile": "p"}})
    assert bench.recorded_traffic("w") == 123
    assert bench.recorded_traffic("other") is None
    monkeypatch.setattr(bench, "MEASURED_TRAFFIC", {"w": {"bytes": 123, "sha256": "0" * 64, "profile": "p"}})
    assert bench.recorded_traffic("w") is None
