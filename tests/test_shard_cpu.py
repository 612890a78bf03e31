"""Host logic of the sequence-sharded forward on CPU: the target ranges of the
ranks cover every split once, and summing disjoint score partials over a
world-size-2 gloo group rebuilds the full matrix (the one exchange step)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import attention_free_long_b200 as av


@pytest.mark.parametrize("n", [1, 7, 64, 1536, 1537])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shard_targets_cover_every_split_once(n, world):
    seen = []
    for r in range(world):
        t0, t1 = av.shard_targets(n, world, r)
        assert 0 <= t0 <= t1 <= n
        seen.extend(range(t0, t1))
    assert seen == list(range(n))
    sizes = [av.shard_targets(n, world, r)[1] - av.shard_targets(n, world, r)[0] for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(0)
        full = torch.randn((2, 11, 11), generator=g)
        owner = torch.arange(full.numel()).reshape(full.shape) % world  # a disjoint ownership
        part = torch.where(owner == rank, full, torch.zeros_like(full))
        dist.all_reduce(part)
        q.put((rank, bool(torch.equal(part, full))))
    finally:
        dist.destroy_process_group()


def test_score_partials_all_reduce_to_the_full_matrix():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == {0: True, 1: True}
