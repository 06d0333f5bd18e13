"""GPU parity of fc_chunk_l1_gate against the CPU oracle.

The Euler update must match bitwise; L1_rel to 1e-6 relative (both sides sum
in float64); the recompute mask and f exactly, except for chunks whose
oracle margin |f + L1 - eps| is below 1e-5 (the margin waiver)."""

import json
import os

import numpy as np
import pytest
import torch

import cache_gating_kv_b200 as fc
from cache_gating_kv_b200 import workloads as W
from oracle import flowcache_oracle as O
from tests.gpu_util import gate_gpu

pytestmark = pytest.mark.gpu
MARGIN = 1e-5


def _compare(out_gpu, out_ref, f_prev, step, m, eps):
    xg, fg, lg, mg = out_gpu
    xr, fr, lr, mr = out_ref
    np.testing.assert_array_equal(xg.view(np.uint32), xr.view(np.uint32))
    np.testing.assert_allclose(lg, lr, rtol=1e-6, atol=0)
    for c in range(len(mr)):
        margin = abs(float(np.float32(f_prev[c] + lr[c])) - eps) if step[c] >= m else 1.0
        if margin < MARGIN:
            continue
        assert mg[c] == mr[c], f"chunk {c}: mask {mg[c]} vs {mr[c]}"
        assert fg[c] == pytest.approx(fr[c], rel=1e-6, abs=0), f"chunk {c}"


def test_gate_hand_trace_on_gpu(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "gate_trace_constant.json")))
    N = g["N"]
    f = np.zeros(1, np.float32)
    ws = fc.workspace(fc.fc_gate_workspace_size(1, N))
    for t in range(g["steps"]):
        x = np.full((1, N), g["x"], np.float32)
        v = np.full((1, N), g["v"], np.float32)
        xn, f, l1, mask = gate_gpu(x, v, [g["dt"]], [t], g["m"], g["eps"], f, ws=ws)
        assert l1[0] == np.float32(g["l1"][t])
        assert mask[0] == g["mask"][t]
        assert f[0] == np.float32(g["f"][t])
        assert np.all(xn == np.float32(g["x_next"]))


@pytest.mark.parametrize("name", ["tiny_fp32", "bf16_layer", "bf16_large_head", "full_step_sweep"])
def test_gate_step_parity_on_workloads(name):
    cfg = W.GATE_CONFIGS[name]
    x = W.gate_initial(cfg, seed=0)
    v = W.gate_velocity(cfg, seed=0)
    rng = np.random.default_rng(1)
    ws = fc.workspace(fc.fc_gate_workspace_size(cfg.n_chunks, cfg.N))
    for eps in cfg.eps:
        for gstep in (0, cfg.m, cfg.T // 2 + cfg.stagger * (cfg.n_chunks - 1) // 2):
            step = W.gate_step_counters(cfg, gstep)
            dt = W.gate_dt(cfg, step)
            f = (rng.random(cfg.n_chunks) * eps).astype(np.float32)
            ref = O.gate_step(x, v, dt, step, cfg.m, eps, f)
            got = gate_gpu(x, v, dt, step, cfg.m, eps, f, ws=ws)
            _compare(got, ref, f, step, cfg.m, eps)


def test_gate_trajectory_with_reuse_feedback():
    """tiny workload over all T steps: a recompute draws a fresh velocity, a
    reuse re-applies the cached one; GPU and oracle advance side by side."""
    cfg = W.GATE_CONFIGS["tiny_fp32"]
    eps = cfg.eps[0]
    x_r = x_g = W.gate_initial(cfg, 0)
    f_r = f_g = np.zeros(cfg.n_chunks, np.float32)
    v_cache = W.gate_velocity(cfg, 0, draw=0)
    mask = np.ones(cfg.n_chunks, np.uint8)
    for t in range(cfg.T):
        fresh = W.gate_velocity(cfg, 0, draw=t)
        v = np.where(mask[:, None] == 1, fresh, v_cache).astype(np.float32)
        v_cache = v
        step = np.full(cfg.n_chunks, t, np.int32)
        dt = W.gate_dt(cfg, step)
        ref = O.gate_step(x_r, v, dt, step, cfg.m, eps, f_r)
        got = gate_gpu(x_g, v, dt, step, cfg.m, eps, f_g)
        _compare(got, ref, f_r, step, cfg.m, eps)
        x_r, f_r, _, mask = ref
        x_g, f_g = got[0], got[1]
        np.testing.assert_array_equal(got[3], mask)


@pytest.mark.parametrize("n_c,N", [(1, 1), (3, 5), (5, 1001), (2, 3), (7, 4099), (1, 0),
                                     (3, 28684), (40, 4096), (2, 4096 * 37 + 64)])
def test_gate_ragged_and_misaligned_chunks(n_c, N):
    rng = np.random.default_rng(N + n_c)
    x = rng.standard_normal((n_c, N)).astype(np.float32)
    v = rng.standard_normal((n_c, N)).astype(np.float32)
    dt = rng.uniform(-0.1, 0.1, n_c).astype(np.float32)
    step = np.arange(n_c, dtype=np.int32)
    f = (rng.random(n_c) * 0.1).astype(np.float32)
    ref = O.gate_step(x, v, dt, step, 1, 0.3, f)
    got = gate_gpu(x, v, dt, step, 1, 0.3, f)
    _compare(got, ref, f, step, 1, 0.3)


def test_gate_inactive_zero_norm_and_forced_steps():
    N = 4096
    x = np.stack([np.ones(N), np.zeros(N), np.zeros(N), np.ones(N), np.ones(N)]).astype(np.float32)
    v = np.stack([np.ones(N), np.ones(N), np.zeros(N), np.ones(N), np.ones(N)]).astype(np.float32)
    dt = np.float32([0.5, 0.5, 0.5, 0.5, 1e-4])
    step = np.int32([-1, 7, 7, 7, 2])
    f = np.float32([0.5, 0.0, 0.0, 0.25, 0.4])
    ref = O.gate_step(x, v, dt, step, 3, 100.0, f)
    got = gate_gpu(x, v, dt, step, 3, 100.0, f)
    _compare(got, ref, f, step, 3, 100.0)
    assert np.isinf(got[2][1]) and got[3][1] == 1
    assert got[2][0] == 0 and got[3][0] == 0 and got[1][0] == np.float32(0.5)
    assert got[3][4] == 1 and got[1][4] == 0  # step 2 < m = 3: forced


def test_gate_deterministic_and_counters_reset():
    cfg = W.GATE_CONFIGS["bf16_layer"]
    x = W.gate_initial(cfg, 3)
    v = W.gate_velocity(cfg, 3)
    step = np.full(cfg.n_chunks, 10, np.int32)
    dt = W.gate_dt(cfg, step)
    f = np.zeros(cfg.n_chunks, np.float32)
    ws = fc.workspace(fc.fc_gate_workspace_size(cfg.n_chunks, cfg.N))
    a = gate_gpu(x, v, dt, step, cfg.m, 0.01, f, ws=ws)
    b = gate_gpu(x, v, dt, step, cfg.m, 0.01, f, ws=ws)
    for u, w in zip(a, b):
        np.testing.assert_array_equal(u, w)
    assert int(ws[: 4 * (cfg.n_chunks + 1)].sum()) == 0  # counters back at zero, no error


# ---------------------------------------------------------------------------
# history-guided gate (fc_history_l1_gate)
# ---------------------------------------------------------------------------
def test_history_gate_hand_trace_on_gpu(golden_dir):
    from tests.gpu_util import history_gate_gpu
    g = json.load(open(os.path.join(golden_dir, "history_gate_trace.json")))
    N = g["N"]
    f = np.zeros(1, np.float32)
    for t in range(g["steps"]):
        h_old = np.full((1, N), g["h_old"], np.float32)
        h_new = np.full((1, N), g["h_new"], np.float32)
        hn, f, d, mask = history_gate_gpu(h_old, h_new, [t], g["m"], g["delta"], f)
        assert d[0] == np.float32(g["d"]) and mask[0] == g["mask"][t] and f[0] == np.float32(g["f"][t])
        assert np.all(hn == np.float32(g["h_new"]))


@pytest.mark.parametrize("n,N", [(4, 777600), (3, 1001), (5, 4096), (16, 24 * 45 * 45 * 16 // 8)])
def test_history_gate_trajectory_parity(n, N):
    """History snapshots drifting over 12 steps; GPU and oracle side by side."""
    from tests.gpu_util import history_gate_gpu
    rng = np.random.default_rng(n * 7 + N)
    h_r = h_g = rng.standard_normal((n, N)).astype(np.float32)
    f_r = f_g = np.zeros(n, np.float32)
    delta = 0.05
    ws = fc.workspace(fc.fc_gate_workspace_size(n, N))
    for t in range(12):
        h_new = (h_r + rng.standard_normal((n, N)).astype(np.float32) *
                 np.float32(0.004 * (1 + t % 3))).astype(np.float32)
        step = np.where(np.arange(n) == n - 1, -1 if t < 3 else t - 3, t).astype(np.int32)
        ref = O.history_gate_step(h_r, h_new, step, 1, delta, f_r)
        got = history_gate_gpu(h_g, h_new, step, 1, delta, f_g, ws=ws)
        np.testing.assert_array_equal(got[0].view(np.uint32), ref[0].view(np.uint32))
        np.testing.assert_allclose(got[2], ref[2], rtol=1e-6)
        for c in range(n):
            margin = abs(float(np.float32(f_r[c] + ref[2][c])) - delta) if step[c] >= 1 else 1.0
            if margin < MARGIN:
                continue
            assert got[3][c] == ref[3][c] and got[1][c] == pytest.approx(ref[1][c], rel=1e-6)
        h_r, f_r = ref[0], ref[1]
        h_g, f_g = got[0], got[1]


def test_full_step_sweep_gate_trajectory_with_reuse_feedback():
    """The 16-chunk full-step-sweep gate over its whole staggered schedule:
    chunk c starts at global step 3c and takes T=50 steps, so global steps
    0..94.  A chunk marked for recompute evaluates the toy's closed-form
    optimal velocity at its current latent, v = (x0 - X)/(1 - sigma(t)) for
    the single-point data x0 (sigma(t) = (t/T)^2); a chunk marked for reuse
    re-applies its cached velocity.  GPU and oracle advance side by side:
    X bitwise at every step, L1 to 1e-6 relative, mask and f exactly outside
    the margin waiver (a waived disagreement re-seeds the GPU side from the
    oracle's state, so that both keep following one trajectory)."""
    cfg = W.GATE_CONFIGS["full_step_sweep"]
    eps = cfg.eps[0]
    n_c = cfg.n_chunks
    x_r = W.gate_initial(cfg, 0)
    x_g = x_r.copy()
    # the toy's data point per chunk: v_exact = x0 - noise, noise = X at t = 0
    x0 = (W.gate_velocity(cfg, 0).astype(np.float64) + x_r.astype(np.float64))
    f_r = np.zeros(n_c, np.float32)
    f_g = f_r.copy()
    v_cache = np.zeros_like(x_r)
    mask = np.ones(n_c, np.uint8)  # a chunk's first step always evaluates the model
    ws = fc.workspace(fc.fc_gate_workspace_size(n_c, cfg.N))
    n_steps = cfg.stagger * (n_c - 1) + cfg.T
    seen_reuse = 0
    waived = 0
    for g in range(n_steps):
        step = W.gate_step_counters(cfg, g)
        dt = W.gate_dt(cfg, step)
        v = v_cache.copy()
        for c in range(n_c):
            if step[c] >= 0 and (mask[c] or step[c] == 0):
                sig = (step[c] / cfg.T) ** cfg.p
                v[c] = ((x0[c] - x_r[c].astype(np.float64)) / (1.0 - sig)).astype(np.float32)
        v_cache = v
        ref = O.gate_step(x_r, v, dt, step, cfg.m, eps, f_r)
        got = gate_gpu(x_g, v, dt, step, cfg.m, eps, f_g, ws=ws)
        np.testing.assert_array_equal(got[0].view(np.uint32), ref[0].view(np.uint32))
        np.testing.assert_allclose(got[2], ref[2], rtol=1e-6, atol=0)
        f_next = got[1].copy()
        for c in range(n_c):
            if step[c] < 0:
                assert got[3][c] == 0 and got[1][c] == f_g[c]
                continue
            margin = abs(float(np.float32(f_r[c] + ref[2][c])) - eps) if step[c] >= cfg.m else 1.0
            if margin < MARGIN:
                if got[3][c] != ref[3][c]:
                    waived += 1
                    f_next[c] = ref[1][c]  # both sides go on from the oracle's decision
                continue
            assert got[3][c] == ref[3][c], f"global step {g}, chunk {c}"
            assert got[1][c] == pytest.approx(ref[1][c], rel=1e-6, abs=0)
        x_r, f_r, _, mask = ref
        seen_reuse += int(np.sum((mask == 0) & (step >= 0)))
        x_g, f_g = got[0], f_next
    assert seen_reuse > 0, "the schedule should reuse some steps at eps = 0.01"
    assert waived <= 2, f"{waived} waived decisions: the margin rule is meant for rare ties"
