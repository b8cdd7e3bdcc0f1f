"""The bench's multi-rank plumbing on CPU: world_size 2 over gloo, replicas only (no data-path
collective): the job time is the max over ranks and the value counts every rank's units."""

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


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import sys

        sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        import bench

        t = bench.max_over_ranks(10.0 + 5.0 * rank, dist, "cpu")  # rank times 10 ms and 15 ms
        v = bench.job_throughput(1e9, 4, world, t)
        out.put((rank, t, v))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, v in res:
        assert t == 15.0  # the slowest replica
        assert v == pytest.approx(1e9 * 4 * 2 / 0.015)  # both ranks' units over the max time


def test_single_process_helpers():
    import bench

    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
    assert bench.job_throughput(100, 2, 1, 1000.0) == 200.0
    cfg = bench.decode_config(4)
    assert cfg["parallelism"].startswith("replicas x4") and cfg["h_kv"] == [32, 8, 1]
