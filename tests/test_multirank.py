"""The bench's multi-rank plumbing on CPU with the gloo backend (world size 2):
max-over-ranks timing, barriers, and the reference arm printing on rank 0
only.  The data path itself has no collective (each rank runs its own copy
of the workload), so nothing else crosses ranks."""
import os
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    bench.barrier(world)
    got = bench.max_over_ranks(1.5 + rank, world)
    out[rank] = got
    bench.barrier(world)
    dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    port = 29500 + (os.getpid() % 2000)
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0] == 2.5 and out[1] == 2.5


def test_reference_arm_non_zero_rank_is_silent():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
