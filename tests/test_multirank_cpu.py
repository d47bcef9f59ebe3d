"""The bench's multi-rank host logic on CPU with gloo (world size 2): each rank runs the same
independent workload, the job time is the slowest rank's, and rank 0 alone reports.  No GPU."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    local_ms = [2.0, 3.0][rank]          # rank 1 is the slow one
    value, ms = bench.aggregate(local_ms, 1e12, world)
    dist.barrier()
    out[rank] = (value, ms)
    dist.destroy_process_group()


def test_aggregate_takes_the_slowest_rank():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    for rank in range(2):
        value, ms = out[rank]
        assert ms == 3.0
        assert abs(value - 2 * 1e12 / 3e-3 / 1e12) < 1e-9


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_aggregate_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    value, ms = bench.aggregate(4.0, 2e12, 1)
    assert ms == 4.0 and abs(value - 500.0) < 1e-9
