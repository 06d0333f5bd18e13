"""The seeded synthetic inputs follow the recipe the parity tests and the bench
rely on: AR(1) key walks with the stated coefficient and stationary variance,
the near-duplicate blocks of the one-layer workload, the exact K/V duplicates
of the long-history workload, the low-rank component of the larger-head
workload, bf16 rounding applied once, the flow-matching toy's velocity, the
gate's step counters and signed steps, and per-head streams that do not depend
on which other heads are drawn."""

import dataclasses

import numpy as np
import torch

from cache_gating_kv_b200 import workloads as W


def _small(name, **kw):
    return dataclasses.replace(W.KV_CONFIGS[name], **kw)


def _lag1(k):
    a, b = k[:-1] - k[:-1].mean(0), k[1:] - k[1:].mean(0)
    return float(((a * b).sum(0) / np.sqrt((a * a).sum(0) * (b * b).sum(0))).mean())


def test_ar1_walk_coefficient_and_variance():
    """tiny_fp32 keys: x_j = 0.9 x_{j-1} + 0.436 n_j, stationary variance
    0.436^2 / (1 - 0.81) = 1.0005; both heads are different walks."""
    cfg = W.KV_CONFIGS["tiny_fp32"]
    _, k0, _ = W.kv_head(cfg, seed=0, head=0)
    _, k1, _ = W.kv_head(cfg, seed=0, head=1)
    for k in (k0, k1):
        assert k.shape == (cfg.Lk, cfg.d) and k.dtype == np.float32
        assert abs(_lag1(k) - 0.9) < 0.03
        assert abs(float(k.var()) - 1.0005) < 0.15
    assert not np.array_equal(k0, k1)


def test_near_duplicate_blocks_of_the_one_layer_workload():
    """In each of the 4 clean chunks the second half is groups of 8 rows that
    are one base plus 0.01-scale noise; the first half is the plain AR walk."""
    cfg = _small("bf16_layer", H=1, Lq=8, Lk=4 * 256)
    _, k, _ = W.kv_head(cfg, seed=3, head=0)
    chunk = cfg.Lk // 4
    for c in range(4):
        lo, mid, hi = c * chunk, c * chunk + chunk // 2, (c + 1) * chunk
        for g0 in range(mid, hi, 8):
            grp = k[g0:g0 + 8]
            spread = np.abs(grp - grp.mean(0)).max()
            assert spread < 0.08, (c, g0, spread)  # 0.01 noise plus bf16 rounding
        first = k[lo:mid]
        steps = np.abs(np.diff(first, axis=0)).mean()
        assert steps > 0.15  # AR(0.95) neighbours differ by ~0.25 per element


def test_exact_duplicates_of_the_long_history_workload():
    """A quarter of the positions copy the K and the V row of another
    position: exactly Lk/4 rows repeat an earlier or later row, and wherever
    two K rows are equal their V rows are equal too."""
    cfg = _small("long_history", H=1, Lq=8, Lk=4096, d=32)
    _, k, v = W.kv_head(cfg, seed=5, head=0)
    _, first, inv = np.unique(k, axis=0, return_index=True, return_inverse=True)
    assert cfg.Lk - len(first) <= cfg.Lk // 4
    counts = np.bincount(inv.ravel())
    copies = int((counts - 1)[counts > 1].sum())
    # every duplicated position is a copy; sources may be copied more than once
    assert copies == cfg.Lk // 4
    for grp in np.flatnonzero(counts > 1)[:200]:
        rows = np.flatnonzero(inv.ravel() == grp)
        assert all(np.array_equal(v[rows[0]], v[r]) for r in rows[1:])


def test_low_rank_component_of_the_larger_head_workload():
    """k = 0.8 ar + 0.6 U z with U in R^{d x 16}: the key covariance has 16
    eigenvalues well above the 0.64 floor of the AR part."""
    cfg = _small("bf16_large_head", H=1, Lq=8, Lk=6000)
    _, k, _ = W.kv_head(cfg, seed=2, head=0)
    ev = np.sort(np.linalg.eigvalsh(np.cov(k.astype(np.float64).T)))[::-1]
    assert ev[:16].mean() > 3.0 * ev[16:].mean()
    assert abs(ev[32:].mean() - 0.64) < 0.15


def test_bf16_workloads_are_rounded_once():
    cfg = _small("bf16_layer", H=1, Lq=64, Lk=512)
    q, k, v = W.kv_head(cfg, seed=0, head=0)
    for a in (q, k, v):
        t = torch.from_numpy(a)
        assert torch.equal(t.to(torch.bfloat16).float(), t)


def test_head_subsets_match_the_full_draw():
    cfg = _small("bf16_layer", H=5, Lq=32, Lk=256)
    Q, K, V = W.kv_inputs(cfg, seed=9)
    q, k, v = W.kv_inputs(cfg, seed=9, heads=[1, 4])
    assert torch.equal(q, Q[[1, 4]]) and torch.equal(k, K[[1, 4]]) and torch.equal(v, V[[1, 4]])
    Q2, _, _ = W.kv_inputs(cfg, seed=10)
    assert not torch.equal(Q2, Q)


def test_flow_matching_toy_velocity_and_steps():
    """x_s = s x0 + (1 - s) eps with X_T the noise: v = x0 - eps, so X + v is
    x0, whose spread is the chunk's x0 standard deviation; dt = sigma(s+1) -
    sigma(s) > 0 with sigma = (t/T)^p; inactive chunks get step -1, dt 0."""
    cfg = dataclasses.replace(W.GATE_CONFIGS["full_step_sweep"], N=20000)
    x = W.gate_initial(cfg, seed=1)
    v = W.gate_velocity(cfg, seed=1)
    assert x.shape == v.shape == (cfg.n_chunks, cfg.N) and x.dtype == v.dtype == np.float32
    for c in range(cfg.n_chunks):
        x0 = x[c].astype(np.float64) + v[c]
        assert abs(x0.std() / cfg.x0_std[c] - 1.0) < 0.03
        assert abs(x[c].std() - 1.0) < 0.03
    st = W.gate_step_counters(cfg, 10)
    np.testing.assert_array_equal(st[:4], [10, 7, 4, 1])
    assert (st[4:] == -1).all()  # chunks 4.. start at global steps 12, 15, ...
    dt = W.gate_dt(cfg, st)
    s = st[:4].astype(np.float64)
    np.testing.assert_allclose(dt[:4], ((s + 1) / cfg.T) ** 2 - (s / cfg.T) ** 2, rtol=1e-6)
    assert (dt[4:] == 0).all()
    late = W.gate_step_counters(cfg, cfg.T - 1 + 3 * 15)  # chunk 15 at its last step
    assert late[0] == -1 and late[15] == cfg.T - 1


def test_gaussian_gate_velocity_redraws_and_scales():
    cfg = W.GATE_CONFIGS["tiny_fp32"]
    v0 = W.gate_velocity(cfg, seed=0, draw=0)
    v1 = W.gate_velocity(cfg, seed=0, draw=1)
    assert not np.array_equal(v0, v1)
    for c, sc in enumerate(cfg.v_scale):
        assert abs(v0[c].std() / sc - 1.0) < 0.05
    np.testing.assert_array_equal(W.gate_dt(cfg, np.zeros(4, np.int32)),
                                  np.full(4, -1.0 / cfg.T, np.float32))


def test_cache_stream_is_one_walk_cut_into_chunks():
    """Consecutive chunks continue the same AR(1) walk: the correlation across
    a chunk boundary is the walk's rho, and each chunk has its own queries."""
    cfg = W.CACHE_CONFIGS["tiny_fp32_ragged"]
    ks, vs, qs = W.cache_inputs(cfg, seed=0)
    assert len(ks) == len(vs) == len(qs) == cfg.n_chunks
    assert ks[0].shape == (cfg.H, cfg.C, cfg.d) and qs[0].shape == (cfg.H, cfg.Lq, cfg.d)
    walk = torch.cat(ks, dim=1)[0].numpy()
    assert abs(_lag1(walk) - cfg.rho) < 0.05
    assert not torch.equal(qs[0], qs[1])
