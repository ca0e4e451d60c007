"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

The W4A4 linear layer shards by tokens with replicated weights and no data
exchange, so the only multi-rank logic is: per-rank batches, the MAX of the
per-rank device times, the whole-job throughput, and rank-0-only output of
the reference arm.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_time = 10.0 + 5.0 * rank          # rank 1 is the slowest
        worst = bench.max_over_ranks(my_time, dist)
        seed = bench.rank_x_seed(rank)
        seeds = [None] * world
        dist.all_gather_object(seeds, seed)
        q.put((rank, worst, seeds))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_seeds():
    port = free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, worst, seeds in res:
        assert worst == 15.0                 # both ranks see the slowest rank's time
        assert len(set(seeds)) == 2          # every replica has its own batch


def test_job_throughput_counts_all_ranks():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.job_throughput(429.5e9, 1, 0.2)
    assert abs(one - 2147.5) < 1e-6
    assert abs(bench.job_throughput(429.5e9, 8, 0.2) - 8 * one) < 1e-6


def test_reference_arm_prints_on_rank0_only(tmp_path):
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
