"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2).

The hot path shards as independent problems per rank (weak scaling): the only
collectives are the timing barrier and one max-reduction of the per-rank
timings. These tests run that reduction over real gloo ranks, check the
per-rank seeding and the whole-job aggregate, and check that the reference
arm runs on rank 0 alone.
"""
import datetime
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from position_remapping_b200.inputs import make_qkv  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sys.path.insert(0, ROOT)
        import bench as b
        # rank r reports times (1 + r, 10 - r, 5): the max is (world, 10, 5)
        dist.barrier()
        got = b.max_over_ranks([1.0 + rank, 10.0 - rank, 5.0], world, "cpu")
        dist.barrier()
        results[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        got = dict(results)
    assert sorted(got) == [0, 1]
    for r in range(world):
        assert got[r] == [2.0, 10.0, 5.0]


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks([3.0, 1.5], 1, "cpu") == [3.0, 1.5]


def test_rank_problems_are_independent_draws():
    seeds = [bench.rank_seed(1004, r) for r in range(8)]
    assert len(set(seeds)) == 8 and seeds[0] == 1004
    a = make_qkv(1, 64, 2, 1, 64, seeds[0])
    b = make_qkv(1, 64, 2, 1, 64, seeds[1])
    a2 = make_qkv(1, 64, 2, 1, 64, seeds[0])
    for x, y, x2 in zip(a, b, a2):
        assert not torch.equal(x, y)
        assert torch.equal(x, x2)


def test_job_throughput_is_weak_scaling_aggregate():
    # N ranks each doing F FLOPs per step for K steps in T ms (slowest rank)
    F, K, T = 1.0e12, 4, 2000.0
    one = bench.job_tflops(1, F, K, T)
    assert one == pytest.approx(F * K / 2.0 / 1e12)
    for n in (2, 4, 8):
        assert bench.job_tflops(n, F, K, T) == pytest.approx(n * one)


def test_reference_arm_runs_on_rank0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
