"""The N > 1 host path of the benchmark on CPU: two gloo ranks agree on the slowest rank's
time, add up the whole job's pairs, draw independent inputs, and the reference arm runs on
rank 0 only."""

import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    bench.init_dist(world, "gloo")
    try:
        w, r, _ = bench.dist_env()
        assert (w, r) == (world, rank)
        slowest = bench.max_over_ranks(10.0 + rank, world)
        total = bench.sum_over_ranks(100 * (rank + 1), world)
        seed = bench.rank_seed(2, rank)
        seeds = [None] * world
        dist.all_gather_object(seeds, seed)
        bench.barrier(world)
        out[rank] = (slowest, total, tuple(seeds))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        slowest, total, seeds = res[rank]
        assert slowest == 11.0            # max over ranks
        assert total == 300.0             # whole-job sum
        assert len(set(seeds)) == world   # independent inputs per rank


def test_reference_arm_runs_on_rank0_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, env=env, timeout=120)
    assert res.returncode == 0 and res.stdout.strip() == ""


def test_cpu_baseline_extrapolation():
    """The CPU baseline's full-step figure scales the sampled rate to the step's pairs."""
    sys.path.insert(0, ROOT)
    import bench
    step = 12 * bench.causal_pairs(200000)
    assert step == 12 * 200000 * 200001 // 2
    assert bench.extrapolated_seconds(step, step // 4, 2.0) == pytest.approx(8.0, rel=1e-12)
    assert bench.extrapolated_seconds(step, 0, 2.0) is None
