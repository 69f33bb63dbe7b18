"""Multi-process host logic of instance sharding, on CPU with the gloo
backend and world size 2 (the GPU launch uses NCCL with the same calls)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from nystr_coreset_approximate_b200 import sharding


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        BH = 33
        lo, hi = sharding.instance_range(BH, world, rank)
        cover = torch.zeros(BH, dtype=torch.int64)
        cover[lo:hi] = 1
        dist.all_reduce(cover)  # every instance owned exactly once
        ms = sharding.max_over_ranks(10.0 + rank)  # per-rank step time -> job time
        x = torch.arange(BH * 2).reshape(BH, 2)
        view, inst0 = sharding.shard(x, world, rank)
        dist.barrier()
        out[rank] = (cover.tolist(), ms, inst0, view[:, 0].tolist())
    finally:
        dist.destroy_process_group()


def test_two_ranks_cover_batch_and_reduce_time():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(world):
        cover, ms, inst0, firsts = res[r]
        assert cover == [1] * 33
        assert ms == 11.0
    assert res[0][2] == 0 and res[1][2] == 17
    assert res[0][3] == [2 * i for i in range(17)]
    assert res[1][3] == [2 * i for i in range(17, 33)]


@pytest.mark.parametrize("BH,world", [(0, 3), (1, 4), (7, 7), (10, 3), (128, 8)])
def test_instance_ranges_partition(BH, world):
    ranges = [sharding.instance_range(BH, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == BH
    assert all(ranges[k][1] == ranges[k + 1][0] for k in range(world - 1))
    sizes = [hi - lo for lo, hi in ranges]
    assert max(sizes) - min(sizes) <= 1


def test_bad_rank_rejected():
    with pytest.raises(ValueError):
        sharding.instance_range(4, 2, 2)
