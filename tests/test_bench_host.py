"""Host logic of the benchmark's multi-GPU path, run as two gloo ranks on the CPU:
the shard split (weak scaling, every rank converts its own sequences, no
collective on the data path) and the max-over-ranks reduction of step times."""
from __future__ import annotations

import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


@pytest.mark.parametrize("total,world", [(4, 1), (4, 2), (7, 2), (32, 3), (5, 8), (0, 2)])
def test_shard_range_partitions(total, world):
    seen = []
    for r in range(world):
        lo, hi = bench.shard_range(total, r, world)
        assert 0 <= lo <= hi <= total
        seen.extend(range(lo, hi))
    assert seen == list(range(total))
    sizes = [bench.shard_range(total, r, world)[1] - bench.shard_range(total, r, world)[0] for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(1.5 + 2.0 * rank)
        lo, hi = bench.shard_range(8, rank, world)
        q.put((rank, got, lo, hi))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [3.5, 3.5]
    assert [(r[2], r[3]) for r in res] == [(0, 4), (4, 8)]


def test_max_over_ranks_without_group():
    assert bench.max_over_ranks(2.25) == 2.25
