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


@pytest.mark.timeout(600)
def test_bench_gpus_flag_launches_replicas_itself():
    """`bench.py --gpus 2` started without torchrun's environment re-launches
    itself under torch.distributed.run with two processes; rank 0 prints the
    one JSON line with n_gpus = 2 (reference arm: CPU only, the other rank
    exits without work)."""
    import json
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR",
                                                            "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--impl", "reference",
                        "--config", "doc8k", "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                       timeout=580, cwd=root, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["impl"] == "reference"


def test_relaunch_command_shape():
    import bench

    cmd = bench.relaunch_command(["--gpus", "4", "--steps", "3"], 4, 29555)
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert "--nproc-per-node=4" in cmd and "127.0.0.1" in cmd and "--master-port=29555" in cmd
    assert cmd[-3:] == ["--gpus", "4", "--steps", "3"] or cmd[-4:] == ["--gpus", "4", "--steps", "3"]
