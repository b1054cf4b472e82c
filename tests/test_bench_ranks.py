"""The multi-process path of bench.py on CPU: two gloo ranks (one process per
GPU on a B200 node, replicas only) agree on the job's time as the slowest
rank's, and the whole-job rate counts every replica's tokens."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out_q):
    import datetime

    import torch.distributed as dist

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.max_over_ranks(dist, times[rank], "cpu")
        out_q.put((rank, got, bench.job_rate(world, 10, 1, got[0])))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_rank_time():
    import torch.multiprocessing as mp

    world, port = 2, _free_port()
    times = [[120.0, 150.0], [100.0, 175.0]]          # per rank: device ms, end-to-end ms
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict()
    for _ in range(world):
        rank, got, rate = q.get(timeout=120)
        results[rank] = (got, rate)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        got, rate = results[rank]
        assert got == [120.0, 175.0]                   # max over ranks, each value
        assert rate == pytest.approx(2 * 10 * 1 / 0.120)  # 20 tokens over the slowest 120 ms


def test_single_process_keeps_its_own_time():
    import bench

    assert bench.max_over_ranks(None, [3.0, 4.5], "cpu") == [3.0, 4.5]
    assert bench.job_rate(1, 2000, 1, 1000.0) == pytest.approx(2000.0)
