"""The multi-GPU host logic on CPU: two gloo ranks agree on the KV-head
shards (disjoint, covering, balanced) and on the max-over-ranks timing the
benchmark reports."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from permuted_block_sparse_b200 import shard


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        lo, hi = shard.kv_head_range(8, world, rank)
        got = [None] * world
        dist.all_gather_object(got, (lo, hi))
        times = shard.max_over_ranks([1.0 + rank, 5.0 - rank], dist)
        q.put((rank, got, times))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_gloo_shards_and_max_timing(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, times in res:
        assert got == [(0, 4), (4, 8)]
        assert times == [2.0, 5.0]                 # max over ranks of (1+r, 5-r)


def test_head_ranges_cover_disjointly():
    for Hkv in (1, 2, 7, 8, 13):
        for world in (1, 2, 3, 4, 8):
            if world > Hkv:
                continue
            ranges = [shard.kv_head_range(Hkv, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == Hkv
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [h - l for l, h in ranges]
            assert max(sizes) - min(sizes) <= 1
    assert shard.query_head_range(32, 8, 4, 1) == (8, 16)
    with pytest.raises(ValueError):
        shard.kv_head_range(8, 2, 2)
