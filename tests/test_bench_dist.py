"""Multi-rank host logic of bench.py on CPU with the gloo backend (world size 2).

Each rank runs its own token batch (weak scaling) with no data-path collective; the timed
region's time is the max over ranks and the reported rate is all ranks' tokens over that
time.  The oracle arm under torchrun prints from rank 0 only.
"""
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
    ms_max = bench.max_over_ranks(ms, world, torch.device("cpu"))
    rate = bench.whole_job_rate(world, 4608, 100, ms_max)
    q.put((rank, ms_max, rate))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_rate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, ms_max, rate in out:
        assert ms_max == 15.0
        assert rate == pytest.approx(2 * 4608 * 100 / 0.015)


def test_reference_arm_prints_only_on_rank_zero():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
