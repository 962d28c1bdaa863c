"""The bench's multi-rank bookkeeping on CPU with two gloo ranks: the step time is the
maximum over ranks, the job throughput counts every rank's work, and only rank 0 of the
reference arm prints (the other ranks exit without work)."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [1.5, 4.0][rank]
        out[rank] = bench.max_over_ranks(local_ms, dist)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_step_time_is_max_over_two_gloo_ranks():
    port = _free_port()
    out = mp.Manager().dict()
    mp.start_processes(_rank_main, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert out[0] == out[1] == 4.0


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_throughput(2, 1e12, 1000.0, 1e12) == pytest.approx(2.0)
    assert bench.max_over_ranks(3.0, None) == 3.0


def test_reference_arm_nonzero_rank_exits_silently():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--gpus", "2"], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
