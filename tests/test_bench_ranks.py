"""The multi-rank host logic of bench.py on CPU (gloo, world size 2).

With N > 1 the benchmark runs N independent replicas; its time is the max of
the per-rank device times and its throughput counts every rank's atoms. The
reference arm prints from rank 0 only.
"""
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank 1 is the slow one: every rank must report its time
        t = bench.max_over_ranks(10.0 + 5.0 * rank, "cpu")
        out[rank] = (t, bench.replica_throughput(world, 512, 20, t))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_replica_throughput():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(2, 29571, out), nprocs=2, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    # 2 replicas x 512 atoms x 20 steps in 15 ms
    assert res[0][1] == pytest.approx(2 * 512 * 20 / 0.015)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, "cpu") == 3.5


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                       env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
