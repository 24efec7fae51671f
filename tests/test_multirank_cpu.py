"""The multi-GPU path of the benchmark shards nothing: each rank runs its own
layer instance (weak scaling) and the only collective is the max of the ranks'
device times.  These tests run that aggregation with two gloo ranks on CPU."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        total = bench.max_over_ranks(times[rank], world, "cpu")
        dist.barrier()
        out[rank] = (total, bench.job_throughput(2048, 10, world, total))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        times = [12.5, 20.0]
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, times, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(2):
        total, value = res[r]
        assert total == 20.0                      # the slowest rank times the job
        assert value == 2048 * 10 * 2 / 0.020     # both ranks' tokens over that time


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.0, 1, "cpu") == 3.0
    assert bench.job_throughput(100, 2, 1, 1000.0) == 200.0


def test_reference_arm_line_carries_the_workload_config(capsys):
    """bench.py --impl reference times the oracle on the host and prints one JSON line
    with the same metric, unit and workload config as the GPU arm's line."""
    import argparse
    import json

    from inputs import gen
    args = argparse.Namespace(workload="tiny_fp32", steps=1, warmup=0, gpus=1, cpu_seconds=0.5)
    bench.run_reference(args, 0)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["higher_is_better"] is True and line["value"] > 0
    assert line["config"] == bench.workload_config(gen.WORKLOADS["tiny_fp32"], 1)
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    # other ranks print nothing
    bench.run_reference(args, 1)
    assert capsys.readouterr().out == ""
