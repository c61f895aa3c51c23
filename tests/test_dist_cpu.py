"""Multi-rank host logic of bench.py on CPU: world size 2 over gloo.

Each rank times its own layer (weak scaling); the job value is the slowest
rank's step time divided by the number of ranks. The reference arm runs on
rank 0 only.
"""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    mx = bench.max_over_ranks(1.5 + rank)           # rank 0: 1.5 ms, rank 1: 2.5 ms
    out[rank] = (mx, bench.job_us_per_layer(mx, world))
    dist.destroy_process_group()


def test_max_over_ranks_and_job_value_world_2():
    import torch.multiprocessing as mp
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
        res = dict(out)
    assert res[0] == res[1] == (2.5, 1250.0)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.job_us_per_layer(0.5, 1) == 500.0


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
