"""The bench's multi-rank plumbing on CPU with the gloo backend (world size 2):
the split of the heads over ranks (the operator's (batch, head) pairs are
independent, so each rank runs its own heads and nothing crosses ranks on the
data path), max-over-ranks timing, barriers, and the reference arm printing
on rank 0 only."""
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("H", [1, 2, 16, 32, 33])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_shard_heads_disjoint_and_covering(H, world):
    spans = [bench.shard_heads(H, world, r) for r in range(world)]
    covered = [h for a, b in spans for h in range(a, b)]
    assert covered == list(range(H))             # disjoint, in order, nothing missing
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench as b
    b.barrier(world)
    got = b.max_over_ranks(1.5 + rank, world)
    # every rank's head span, gathered: the union must be all heads, once
    span = torch.tensor(b.shard_heads(32, world, rank))
    spans = [torch.zeros(2, dtype=span.dtype) for _ in range(world)]
    dist.all_gather(spans, span)
    out[rank] = (got, [tuple(s.tolist()) for s in spans])
    b.barrier(world)
    dist.destroy_process_group()


def test_max_over_ranks_and_head_split_gloo():
    world = 2
    port = 29500 + (os.getpid() % 2000)
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == 2.5 and out[1][0] == 2.5
    spans = out[0][1]
    assert spans == out[1][1]
    heads = sorted(h for a, b in spans for h in range(a, b))
    assert heads == list(range(32))


def test_reference_arm_non_zero_rank_is_silent():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
