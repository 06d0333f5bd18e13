"""The zero-exchange split of the path, on the library itself.

`bench.py --shard heads` gives each rank a contiguous range of one layer's
heads and of the gate's chunks (every head and every chunk is independent, so
nothing is exchanged).  Here the ranges of 2, 3 and 5 ranks run one after
another on one GPU, and the pieces put together are compared with the calls
over the whole layer:

- redundancy, score/top-B and compaction: bitwise (each head is one cluster
  or one independent row of work whatever the head count);
- importance: within 2e-6 relative; the row pass picks its key split from
  the grid size, which depends on the number of heads in the call, and a
  different split adds the same exponentials in another order;
- the selection of each piece, re-run over the whole layer's scores: bitwise;
  the whole-layer selection against the pieces': identical up to the margin
  waiver of the importance's rounding;
- gate: the Euler update bitwise, L1 to 1e-7 relative (the blocks per chunk
  depend on the chunk count), masks and accumulators exact outside the
  margin waiver.
"""

import numpy as np
import pytest
import torch

import bench
import cache_gating_kv_b200 as fc
from cache_gating_kv_b200 import workloads as W
from tests.gpu_util import (assert_selection_matches, compact_gpu, gate_gpu, importance_gpu,
                            redundancy_gpu, score_topb_gpu)

pytestmark = pytest.mark.gpu
MARGIN = 1e-5


def _layer(q, k, v, cfg, lam):
    imp = importance_gpu(q, k)
    red = redundancy_gpu(k)
    sc, idx = score_topb_gpu(imp, red, cfg.pool, lam, cfg.B)
    ko, vo = compact_gpu(k, v, idx)
    return imp, red, sc, idx, ko, vo


@pytest.mark.parametrize("name", ["bf16_layer", "bf16_large_head"])
@pytest.mark.parametrize("world", [2, 3, 5])
def test_head_shards_rebuild_the_layer(name, world):
    cfg = W.KV_CONFIGS[name]
    q, k, v = W.kv_inputs(cfg, seed=0)
    lam = cfg.lam[len(cfg.lam) // 2]
    whole = _layer(q, k, v, cfg, lam)
    parts = []
    for r in range(world):
        lo, hi = bench.shard_heads(cfg.H, r, world)
        parts.append(_layer(q[lo:hi], k[lo:hi], v[lo:hi], cfg, lam))
    imp, red, sc, idx = (np.concatenate([p[i] for p in parts]) for i in range(4))
    ko = torch.cat([p[4] for p in parts])
    vo = torch.cat([p[5] for p in parts])
    np.testing.assert_allclose(imp, whole[0], rtol=2e-6, atol=0)
    np.testing.assert_array_equal(red.view(np.uint32), whole[1].view(np.uint32))
    # the selection is per head: run over the whole layer on the pieces' own
    # Imp and Red it gives the pieces' scores and indices bitwise
    sc2, idx2 = score_topb_gpu(imp, red, cfg.pool, lam, cfg.B)
    np.testing.assert_array_equal(sc2.view(np.uint32), sc.view(np.uint32))
    np.testing.assert_array_equal(idx2, idx)
    ko2, vo2 = compact_gpu(k, v, idx)
    assert torch.equal(ko2, ko) and torch.equal(vo2, vo)
    # and against the whole-layer selection, up to the importance's rounding
    span = (whole[2].max(axis=1) - whole[2].min(axis=1)).max()
    assert_selection_matches(idx, whole[2].astype(np.float64), cfg.B, 1e-5 * span)


@pytest.mark.parametrize("name", ["bf16_layer", "bf16_large_head", "full_step_sweep"])
@pytest.mark.parametrize("world", [2, 3, 5])
def test_chunk_shards_rebuild_the_gate(name, world):
    cfg = W.GATE_CONFIGS[name]
    x = W.gate_initial(cfg, 0)
    v = W.gate_velocity(cfg, 0)
    g = cfg.m + 2 + cfg.stagger * (cfg.n_chunks - 1) // 2
    step = W.gate_step_counters(cfg, g)
    dt = W.gate_dt(cfg, step)
    f = (np.random.default_rng(world).random(cfg.n_chunks) * cfg.eps[0]).astype(np.float32)
    eps = cfg.eps[0]
    xw, fw, lw, mw = gate_gpu(x, v, dt, step, cfg.m, eps, f)
    pieces = []
    for r in range(world):
        lo, hi = bench.shard_heads(cfg.n_chunks, r, world)
        if hi > lo:
            pieces.append(gate_gpu(x[lo:hi], v[lo:hi], dt[lo:hi], step[lo:hi], cfg.m, eps,
                                   f[lo:hi]))
    xs, fs, ls, ms = (np.concatenate([p[i] for p in pieces]) for i in range(4))
    np.testing.assert_array_equal(xs.view(np.uint32), xw.view(np.uint32))
    np.testing.assert_allclose(ls, lw, rtol=1e-7, atol=0)
    for c in range(cfg.n_chunks):
        if step[c] >= cfg.m and abs(float(np.float32(f[c] + lw[c])) - eps) < MARGIN:
            continue
        assert ms[c] == mw[c] and fs[c] == pytest.approx(fw[c], rel=1e-7, abs=0), c
