"""Host logic of the N > 1 bench path on CPU with 2 gloo ranks: every rank
owns a disjoint slice of the global batch, the slices cover it exactly once,
and the step time reported is the max over ranks."""
import os

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _worker(rank, world, port, global_batch, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lo, hi = bench.rank_batch_slice(global_batch, world, rank)
        mine = torch.zeros(global_batch, dtype=torch.int64)
        mine[lo:hi] = 1
        dist.all_reduce(mine)
        t = bench.max_over_ranks(1.0 + rank * 0.25)
        out.put((rank, lo, hi, mine.tolist(), t))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("global_batch", [2, 5, 8])
def test_two_rank_sharding_and_max_time(global_batch):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + global_batch + os.getpid() % 500
    procs = [ctx.Process(target=_worker, args=(r, 2, port, global_batch, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][2] == res[1][1] and res[0][1] == 0 and res[1][2] == global_batch
    assert res[0][3] == [1] * global_batch          # every batch row owned exactly once
    assert res[0][4] == res[1][4] == 1.25            # max over ranks


def test_single_process_identity():
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.rank_batch_slice(7, 1, 0) == (0, 7)
    sizes = [bench.rank_batch_slice(10, 4, r) for r in range(4)]
    assert sizes == [(0, 3), (3, 6), (6, 8), (8, 10)]
