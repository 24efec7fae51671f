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
