"""Repeated runs are bitwise identical: every reduction has a fixed order and
no call uses floating-point atomics, so a difference between two runs would
point at a race.  Covers the importance (with its key split), the
redundancy, score/top-B, compaction, the gate and the cache commit on
workload-sized inputs."""

import numpy as np
import pytest
import torch

import cache_gating_kv_b200 as fc
from cache_gating_kv_b200 import workloads as W
from tests.gpu_util import DEV

pytestmark = pytest.mark.gpu


def _run_chain(q, k, v, B):
    H, Lq, d = q.shape
    Lk = k.shape[1]
    imp = torch.empty(H, Lk, device=DEV)
    red = torch.empty(H, Lk, device=DEV)
    sc = torch.empty(H, Lk, device=DEV)
    idx = torch.empty(H, B, dtype=torch.int32, device=DEV)
    ko = torch.empty(H, B, d, dtype=k.dtype, device=DEV)
    vo = torch.empty_like(ko)
    fc.fc_kv_importance(q, k, imp, fc.workspace(fc.fc_importance_workspace_size(fc.FC_BF16, H, Lq,
                                                                                 Lk, d)))
    fc.fc_kv_redundancy(k, red, fc.workspace(fc.fc_redundancy_workspace_size(fc.FC_BF16, H, Lk, d)))
    fc.fc_kv_score_topb(imp, red, 7, 0.5, B, idx,
                        fc.workspace(fc.fc_score_topb_workspace_size(H, Lk, B)), score=sc)
    fc.fc_kv_compact(k, v, idx, ko, vo)
    torch.cuda.synchronize()
    return [t.cpu() for t in (imp, red, sc, idx, ko, vo)]


def test_compression_chain_is_bitwise_repeatable():
    cfg = W.KV_CONFIGS["bf16_layer"]
    q, k, v = W.kv_inputs(cfg, seed=4, heads=range(6))
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    a = _run_chain(q, k, v, cfg.B)
    b = _run_chain(q, k, v, cfg.B)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


def test_gate_is_bitwise_repeatable():
    cfg = W.GATE_CONFIGS["full_step_sweep"]
    x0 = torch.from_numpy(W.gate_initial(cfg, 0))
    v = torch.from_numpy(W.gate_velocity(cfg, 0)).to(DEV)
    st = torch.full((cfg.n_chunks,), cfg.m + 1, dtype=torch.int32, device=DEV)
    dt = torch.full((cfg.n_chunks,), -0.01, device=DEV)
    outs = []
    for _ in range(2):
        x = x0.to(DEV)
        f = torch.zeros(cfg.n_chunks, device=DEV)
        l1 = torch.empty(cfg.n_chunks, device=DEV)
        mask = torch.empty(cfg.n_chunks, dtype=torch.uint8, device=DEV)
        ws = fc.workspace(fc.fc_gate_workspace_size(cfg.n_chunks, cfg.N))
        fc.fc_chunk_l1_gate(x, v, dt, st, cfg.m, 0.01, f, l1, mask, ws)
        torch.cuda.synchronize()
        outs.append([t.cpu() for t in (x, f, l1, mask)])
    for p, r in zip(*outs):
        assert torch.equal(p.view(torch.uint8), r.view(torch.uint8))


def test_cache_commit_is_bitwise_repeatable():
    cfg = W.CACHE_CONFIGS["bf16_stream"]
    ks, vs, qs = W.cache_inputs(cfg, seed=5)
    H, C, B, d = cfg.H, cfg.C, cfg.B_budget, cfg.d
    kb = torch.cat(ks[:5], dim=1).to(DEV)
    vb = torch.cat(vs[:5], dim=1).to(DEV)
    q = qs[5].to(DEV)
    outs = []
    for _ in range(2):
        kn, vn = torch.zeros_like(kb), torch.zeros_like(vb)
        idx = torch.empty(H, B, dtype=torch.int32, device=DEV)
        ws = fc.workspace(fc.fc_kv_cache_workspace_size(fc.FC_BF16, H, cfg.Lq, B, C, d))
        n, comp = fc.fc_kv_cache_commit(q, kb, vb, kn, vn, B, C, ws, cfg.pool, cfg.lam, idx=idx)
        torch.cuda.synchronize()
        assert comp and n == B
        outs.append([t.cpu() for t in (kn, vn, idx)])
    for p, r in zip(*outs):
        assert torch.equal(p.view(torch.uint8), r.view(torch.uint8))


def test_step_soak_replays_bitwise():
    """The bench's one-layer step (gate and redundancy on a second stream
    beside the importance) captured once and replayed 200 times: every replay
    gives the first replay's outputs bitwise, and no bounded wait gives up."""
    import bench

    dev = torch.device(DEV, torch.cuda.current_device())
    kv_cfg, gate_cfg = bench.configs("bf16_layer")
    step = bench.Step(kv_cfg, gate_cfg, seed=0, dev=dev)
    main = torch.cuda.Stream(device=dev)
    side = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(main):
        step.run(main, side=side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=main, capture_error_mode="relaxed"):
            step.run(main, side=side)
        names = ("imp", "red", "idx", "ko", "vo")
        first = None
        for i in range(200):
            step.d["x"].copy_(step.host["x"].to(dev))  # the gate updates X in place
            step.d["f"].zero_()
            g.replay()
            main.synchronize()
            if i % 20 == 0 or i == 199:
                cur = [step.out[n].clone() for n in names] + [step.d["x"].clone()]
                if first is None:
                    first = cur
                else:
                    for a, b in zip(first, cur):
                        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), f"replay {i}"
        del g
    assert fc.fc_check_workspace(fc.FC_WS_IMPORTANCE, step.ws["imp"])
