"""Multi-rank host logic of the benchmark on CPU: two gloo ranks, the way
torchrun launches the replicas (one process per GPU on the box).  No GPU and no
kernel runs here; the layer needs no collective, so what is checked is the
rank bookkeeping: the max-over-ranks timing, the whole-job rate and the
reference arm's rank-0-only output."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took (r + 1) * 10 ms; every rank must see the slowest one
        slowest = bench.max_over_ranks(10.0 * (rank + 1), world, torch.device("cpu"))
        rate = bench.whole_job_rate(21, 100, world, slowest)
        out[rank] = (slowest, rate)
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_count_all_units():
    world = 2
    port = 29500 + (os.getpid() % 1000)
    with mp.Manager() as man:
        out = man.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == pytest.approx(20.0) and res[1][0] == pytest.approx(20.0)
    # 21 tokens per step per replica, 100 steps, 2 replicas, in the slowest rank's 20 ms
    assert res[0][1] == pytest.approx(21 * 100 * 2 / 0.020)


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r1 = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                         "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r1.returncode == 0
    assert r1.stdout.strip() == ""
    env.update(RANK="0", LOCAL_RANK="0")
    r0 = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                         "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r0.returncode == 0
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
