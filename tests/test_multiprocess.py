"""Replica host logic of bench.py under torch.distributed with world size 2
(gloo on CPU): the max-over-ranks time and the whole-job throughput that
rank 0 reports.  The attention path has no exchange step, so no data-path
collective exists to test; only the timing aggregation is shared."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    from datetime import timedelta

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench

    local_ms = [100.0, 250.0][rank]
    value, total = bench.aggregate(local_ms, flops_per_step=1e12, steps=10, world=world, device="cpu")
    bench.barrier(world)
    out[rank] = (value, total)
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_replicas_report_whole_job_throughput():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    # every rank sees the max time; value = all ranks' FLOPs / that time
    for r in range(world):
        value, total = out[r]
        assert total == 250.0
        assert abs(value - world * 1e12 * 10 / 0.25 / 1e12) < 1e-9


def test_single_rank_aggregate():
    import bench

    v, t = bench.aggregate(500.0, 2e12, 5, 1, "cpu")
    assert t == 500.0 and abs(v - 20.0) < 1e-12
