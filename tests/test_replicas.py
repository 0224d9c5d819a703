"""Multi-process host logic of bench.py on the CPU (gloo, world size 2).

The convolution does not shard (one GPU, no collective); N GPUs run N
independent replicas.  What needs checking without GPUs is the host side:
the max-over-ranks timing, the whole-job aggregate, and that the reference arm
prints only on rank 0.
"""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    t = 10.0 + 5.0 * rank                      # rank 1 is the slow one
    t_max = bench.reduce_max(t, world)
    dist.barrier()
    out[rank] = (t_max, bench.aggregate_gbs(1_000_000_000, 4, world, t_max))
    dist.destroy_process_group()


def test_max_over_ranks_and_aggregate():
    world = 2
    port = 29600 + os.getpid() % 300
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    # 2 ranks x 4 steps x 1 GB over 15 ms
    assert abs(res[0][1] - 2 * 4 * 1.0 / 0.015) < 1e-6


def test_reference_arm_prints_only_on_rank_zero():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


@pytest.mark.slow
def test_reference_arm_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "2", "--warmup", "3", "--ref-seconds", "5"], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"
