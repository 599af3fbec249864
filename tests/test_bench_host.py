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


def test_emitted_line_carries_the_contract_keys(capsys):
    # the JSON line the driver parses: every key and its type, built from fake measurements
    import json
    from types import SimpleNamespace
    import bench
    from block_sparse_long_scores_b200.workloads import WORKLOADS

    w = WORKLOADS["prefill_128k"]
    roofline = {"bound": "tensor", "achieved": 400.0, "peak": 1414.8, "unit": "TFLOP/s", "frac": 400.0 / 1414.8,
                "traffic": 9.9e9}
    cpu = {"value": 300.0, "unit": "tokens/s", "cores": 16, "kind": "oracle", "sample": "rows"}
    e2e = {"value": 1.5e6, "unit": "tokens/s", "h2d_bytes_per_step": 1, "d2h_bytes_per_step": 1}
    clk = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    bench.emit(SimpleNamespace(steps=5, warmup=3), SimpleNamespace(rank=0, world=1), w, 131072,
               16384, 3.1e6, 41.5, roofline, cpu, e2e, 325, clk, 213.0, {}, {})
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key, typ in [("metric", str), ("value", float), ("unit", str), ("n_gpus", int), ("steps", int),
                     ("warmup", int), ("ms_per_step", float), ("higher_is_better", bool), ("scaling", str),
                     ("dtype", str), ("data", str), ("config", dict), ("roofline", dict), ("cpu_baseline", dict),
                     ("e2e", dict), ("gpu_launches", int), ("clocks", dict)]:
        assert isinstance(line[key], typ), key
    assert "vs_baseline" in line and line["scaling"] == "weak" and line["higher_is_better"] is True
    assert set(roofline) <= set(line["roofline"]) and line["cpu_baseline"]["kind"] == "oracle"
    assert {"workload", "global_batch", "seq_len", "l2"} <= set(line["config"])
    assert "1.07 GB" in line["config"]["l2"] and "+ sink" in line["config"]["workload"]
    # the ragged workload has no sink and unequal lengths
    wr = WORKLOADS["ragged_prefill"]
    bench.emit(SimpleNamespace(steps=1, warmup=1), SimpleNamespace(rank=0, world=1), wr, sum(wr.seqlens),
               16384, 1.0, 1.0, roofline, None, None, 1, clk, 1.0, {}, {})
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert "+ sink" not in line["config"]["workload"] and "(ragged)" in line["config"]["workload"]


def test_both_arms_describe_the_same_config():
    import bench
    from block_sparse_long_scores_b200.workloads import WORKLOADS
    w = WORKLOADS["prefill_128k"]
    ours = bench.workload_config(w, 131072, 16384, 1)
    ref = bench.workload_config(w, w.total_rows, min(16384, w.total_rows), 1)
    assert ours == ref
