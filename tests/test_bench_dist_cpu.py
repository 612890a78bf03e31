"""Host-side logic of the multi-GPU benchmark, on CPU with the gloo backend at
world size 2: every rank encodes its own sequence (distinct seeds, no
data-path collective) and the step time reported is the max over ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist = bench.init_dist("gloo", world)
    try:
        assert bench.dist_env() == (rank, world, rank)
        ms = 10.0 + 5.0 * rank  # rank 1 is slower
        got = bench.max_over_ranks(ms)
        seed = bench.rank_seed(rank)
        q.put((rank, got, seed))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_distinct_sequences():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    res = sorted(q.get(timeout=5) for _ in range(world))
    assert [r[1] for r in res] == [15.0, 15.0]      # both ranks see the slowest rank's time
    assert len({r[2] for r in res}) == world         # one distinct sequence per rank


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5


def test_l2_notes_follow_the_workload():
    import bench
    import synthetic as sy
    assert "larger than L2" in bench.l2_note(sy.WORKLOADS["long_bf16"])
    assert "fits" in bench.l2_note(sy.WORKLOADS["base_bf16"])
    assert "larger than L2" in bench.l2_note(sy.WORKLOADS["large_bf16"])


def test_compress_bytes_count_what_the_forward_writes():
    import bench
    import synthetic as sy
    wl = sy.WORKLOADS["long_bf16"]
    # 8 gathered blocks of bf16 in, the split pair out: 1.51 GB
    assert bench.compress_bytes(wl) == 8 * 98304 * 768 * 2 + 98304 * 768 * 4
    no_layers = sy.custom("c0", B=1, N=1024, S=64, d=64, m=128, k=3, pattern=())
    assert bench.compress_bytes(no_layers) == 4 * 1024 * 64 * 2 + 1024 * 64 * 8
