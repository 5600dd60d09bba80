"""The benchmark's multi-rank plumbing on CPU with the gloo backend.

bench.py runs one replica of the workload per GPU (the problems are
independent, so there is no data-path collective); across ranks it only
takes the max of the timed durations and reports the whole-job throughput.
These tests run that plumbing as two gloo ranks on the CPU."""
import json
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ws, r, lr = bench.dist_env()
        t = bench.reduce_max(1.0 + rank, ws, torch.device("cpu"))
        bench.barrier(ws)
        q.put((rank, ws, r, lr, t))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ws, r, lr, t in out:
        assert ws == 2 and r == rank and lr == rank
        assert t == 2.0  # the slowest rank's time


def test_reference_arm_prints_only_on_rank_zero():
    # the reference arm (the CPU oracle) runs on rank 0 alone; other ranks exit
    # quietly. Rank 1 is simulated through the environment.
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
