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


def _lonely_worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    try:
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=3))
        out[rank] = "joined"
        dist.destroy_process_group()
    except Exception as e:  # the rendezvous ends with an error, not a hang
        out[rank] = type(e).__name__


def test_rank_that_never_joins_ends_in_a_bounded_error():
    import time

    import torch.multiprocessing as mp
    port = _free_port()
    t0 = time.time()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_lonely_worker, args=(2, port, out), nprocs=1, start_method="spawn", join=True)
        res = dict(out)
    assert res[0] != "joined"
    assert time.time() - t0 < 60


def _dying_worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        out[rank] = "left before the step's collective"
        os._exit(3)  # the rank dies between steps, with nothing in flight
    try:
        bench.max_over_ranks(1.0)
        out[rank] = "collective completed"
    except Exception as e:
        out[rank] = type(e).__name__


def test_rank_that_dies_is_seen_by_the_other_rank():
    import torch.multiprocessing as mp
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        ctx = mp.start_processes(_dying_worker, args=(2, port, out), nprocs=2, start_method="spawn", join=False)
        for p in ctx.processes:
            p.join(timeout=60)
        codes = [p.exitcode for p in ctx.processes]
        res = dict(out)
    assert codes[1] == 3
    assert res[1] == "left before the step's collective"
    assert res.get(0) not in (None, "collective completed")
