"""Host logic of the multi-GPU benchmark, on CPU: two gloo ranks stand in for two GPUs.

The path shards into independent sequences (one per rank, no data-path collective); the only
collective is the max over ranks of the measured time, and the whole-job rate divides every
rank's rows by that slowest time.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import bench
    d = bench.Dist(world, backend="gloo")
    d.barrier()
    ms_max = d.max(times[rank])
    value = bench.throughput(d.world, 131072, 5, ms_max)
    out.put((rank, d.world, ms_max, value))
    d.close()


def test_two_rank_max_and_weak_scaling_rate():
    world, port = 2, _free_port()
    times = [120.0, 150.0]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, w, ms_max, value in res:
        assert w == 2 and ms_max == 150.0                       # every rank sees the slowest time
        assert value == pytest.approx(2 * 131072 * 5 / 0.150)   # all ranks' rows / slowest time


def test_single_process_rate():
    import bench
    assert bench.throughput(1, 131072, 5, 250.0) == pytest.approx(131072 * 5 / 0.25)
