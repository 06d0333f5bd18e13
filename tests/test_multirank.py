"""The N > 1 host logic of bench.py on CPU: two gloo ranks agree on the
max-over-ranks timing, the head split covers every head exactly once, and
the head-sharded mode's per-rank inputs put together are the whole layer's."""

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


def _shard_worker(rank, world, port, out):
    from cache_gating_kv_b200 import workloads as W

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        kv_cfg, gate_cfg = bench.configs("tiny_fp32")
        lo, hi = bench.shard_heads(kv_cfg.H, rank, world)
        q, k, v = W.kv_inputs(kv_cfg, seed=0, heads=range(lo, hi))
        parts = [torch.zeros(1, kv_cfg.Lk, kv_cfg.d) for _ in range(world)]
        dist.all_gather(parts, k.float())  # H = world: one head each
        out[rank] = torch.cat(parts).numpy().tobytes()
        clo, chi = bench.shard_heads(gate_cfg.n_chunks, rank, world)
        x = torch.from_numpy(W.gate_initial(gate_cfg, 0)[clo:chi].copy())
        xs = [torch.zeros(chi - clo, gate_cfg.N) for _ in range(world)]
        dist.all_gather(xs, x)
        assert torch.equal(torch.cat(xs), torch.from_numpy(W.gate_initial(gate_cfg, 0)))
    finally:
        dist.destroy_process_group()


def test_head_sharded_inputs_rebuild_the_layer():
    from cache_gating_kv_b200 import workloads as W

    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_shard_worker, args=(world, port, out), nprocs=world, join=True)
        _, k_full, _ = W.kv_inputs(W.KV_CONFIGS["tiny_fp32"], seed=0)
        for r in range(world):
            assert out[r] == k_full.float().numpy().tobytes()


def test_bench_workload_names():
    from cache_gating_kv_b200 import workloads as W

    assert bench.configs("bf16_layer")[1] is W.GATE_CONFIGS["bf16_layer"]
    assert bench.configs("sweep_lk131072")[1] is W.GATE_CONFIGS["full_step_sweep"]
    assert bench.configs("long_history")[1] is None
