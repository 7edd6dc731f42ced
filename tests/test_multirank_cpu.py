"""The multi-rank plumbing of bench.py on CPU (gloo, world size 2): each rank's
timing is reduced as a max, bytes as a sum, every rank draws its own batch, and
the reference arm prints from rank 0 only."""

import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = bench.max_over_ranks(10.0 + rank, world, "cpu")
        b = bench.sum_over_ranks(100.0 * (rank + 1), world, "cpu")
        lens = bench.workloads.uniform_lengths(bench.BATCH, 1, bench.MAX_LEN, 0 + 1000 * rank)
        bench.barrier(world)
        q.put((rank, t, b, lens[:4]))
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_max_time_and_sum_bytes():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [11.0, 11.0]      # the slowest rank's time
    assert [r[2] for r in res] == [300.0, 300.0]    # bytes of both ranks
    assert res[0][3] != res[1][3]                   # independent batches per rank


def test_reference_arm_is_silent_on_other_ranks():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", CUDA_VISIBLE_DEVICES="")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--steps", "1", "--warmup", "3"], env=env,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0
    assert out.stdout.strip() == ""
