"""The N > 1 host logic of bench.py on CPU: two gloo ranks agree on the
max-over-ranks timing, and the head split covers every head exactly once."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.reduce_max([1.0 + rank, 10.0 - rank], world, "cpu")
        out[rank] = got
        lo, hi = bench.shard_heads(40, rank, world)
        t = torch.zeros(40, dtype=torch.int64)
        t[lo:hi] = 1
        dist.all_reduce(t)
        assert torch.equal(t, torch.ones(40, dtype=torch.int64))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_max_over_ranks_and_head_shards(world):
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        for r in range(world):
            assert out[r] == [float(world), 10.0]


def test_shard_heads_single_process():
    for H in (1, 7, 24, 40):
        for world in (1, 2, 3, 8):
            spans = [bench.shard_heads(H, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            assert max(h - l for l, h in spans) - min(h - l for l, h in spans) <= 1
    assert bench.reduce_max([3.0, 4.0], 1, "cpu") == [3.0, 4.0]
