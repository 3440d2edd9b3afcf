"""Multi-rank logic of the benchmark on CPU (gloo, world size 2).

The attention path shards by (b, h) head with no collective; ranks only agree
on timing.  Each rank contributes its own timings and the job's throughput
uses the slowest rank."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        local = [1.0 + rank, 5.0 - rank, 2.5]
        got = bench.max_over_ranks(local, dist, "cpu")
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0] == out[1] == [2.0, 5.0, 2.5]


def test_single_process_is_identity_and_throughput_scales_with_ranks():
    import bench
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    one = bench.whole_job_tflops(1e12, 1, 10.0)
    assert abs(one - 100.0) < 1e-9
    assert abs(bench.whole_job_tflops(1e12, 4, 10.0) - 4 * one) < 1e-9
