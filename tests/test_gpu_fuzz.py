"""Seeded random cases for every call against the oracle: ragged sizes, both
dtypes and head dims, random pooling windows, lambdas (also outside [0, 1]),
budgets (also B >= L_k), explicit softmax scales, cache commits of both dtypes
(any chunk size, fewer candidates than the buffer holds), chunk counts and sizes that
are not multiples of 4, inactive chunks and zero updates.  The tolerances and
margin waivers are the ones the other parity tests use."""

import numpy as np
import pytest
import torch

import cache_gating_kv_b200 as fc
from oracle import flowcache_oracle as O
from tests.gpu_util import (DEV, TOL_BF16, TOL_F32, assert_selection_matches, compact_gpu, f64,
                            gate_gpu, history_gate_gpu, importance_gpu, redundancy_gpu,
                            score_topb_gpu)

pytestmark = pytest.mark.gpu
MARGIN = 1e-5


def _close(got, ref, bf16):
    if bf16:
        atol = 1e-4 * np.abs(ref).max(axis=-1, keepdims=True)
        assert np.all(np.abs(got - ref) <= 1e-4 * np.abs(ref) + atol)
    else:
        np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-9 * np.abs(ref).max())


def _kv_case(seed):
    rng = np.random.default_rng(7000 + seed)
    H = int(rng.integers(1, 5))
    Lq = int(rng.integers(1, 700))
    Lk = int(rng.integers(1, 1800))
    d = int(rng.choice([64, 128]))
    bf16 = bool(rng.integers(0, 2))
    B = int(rng.integers(1, Lk + 20))
    pool = int(rng.choice([1, 3, 5, 7, 15, 63]))
    lam = float(rng.uniform(-0.2, 1.2))
    scale = 0.0 if rng.random() < 0.5 else float(rng.uniform(0.03, 0.3))
    g = torch.Generator().manual_seed(seed)
    dt = torch.bfloat16 if bf16 else torch.float32
    q = torch.randn(H, Lq, d, generator=g).to(dt)
    # keys with some structure: a shared direction and a few exact duplicates
    k = torch.randn(H, Lk, d, generator=g) + 0.5 * torch.randn(H, 1, d, generator=g)
    if Lk > 4:
        k[:, 1::5] = k[:, 0:1]
    k = k.to(dt)
    v = torch.randn(H, Lk, d, generator=g).to(dt)
    return H, Lq, Lk, d, bf16, B, pool, lam, scale, q, k, v


@pytest.mark.parametrize("seed", range(48))
def test_kv_chain_random(seed):
    H, Lq, Lk, d, bf16, B, pool, lam, scale, q, k, v = _kv_case(seed)
    imp = importance_gpu(q, k, scale=scale)
    red = redundancy_gpu(k)
    imp_r = O.importance(f64(q), f64(k), scale=scale if scale > 0 else None)
    red_r = O.redundancy(f64(k))
    _close(imp, imp_r, bf16)
    _close(red, red_r, False)
    sc, idx = score_topb_gpu(imp, red, pool, lam, B)
    sc_r, idx_r = O.score_topb(imp_r, red_r, lam, pool, B)
    tol = TOL_BF16 if bf16 else TOL_F32
    for h in range(H):
        span = (sc_r[h].max() - sc_r[h].min()) if bf16 else np.abs(sc_r[h]).max()
        span = max(float(span), 1e-30)
        assert np.max(np.abs(sc[h] - sc_r[h])) <= tol * span
        if B >= Lk:
            np.testing.assert_array_equal(idx[h], idx_r[h])  # keep-all is exact
        else:
            assert_selection_matches(idx[h:h + 1], sc_r[h:h + 1].astype(np.float64), B,
                                     tol * span)
    ko, vo = compact_gpu(k, v, idx)
    for h in range(H):
        keep = idx[h] >= 0
        sel = torch.from_numpy(idx[h][keep].astype(np.int64))
        assert torch.equal(ko[h][torch.from_numpy(keep)], k[h].index_select(0, sel))
        assert torch.equal(vo[h][torch.from_numpy(keep)], v[h].index_select(0, sel))
        assert not ko[h][torch.from_numpy(~keep)].float().abs().sum().item()


def _gate_case(seed):
    rng = np.random.default_rng(9000 + seed)
    n_c = int(rng.integers(1, 25))
    N = int(rng.choice([0, 1, 3, 5, 4096, 4097, int(rng.integers(1, 60000))]))
    x = (rng.standard_normal((n_c, N)) * rng.uniform(0.1, 3.0)).astype(np.float32)
    v = rng.standard_normal((n_c, N)).astype(np.float32)
    if n_c > 2 and N:
        v[1] = 0.0  # a zero update
        x[2] = 0.0  # a zero state
    step = rng.integers(-1, 9, n_c).astype(np.int32)
    m = int(rng.integers(0, 4))
    eps = float(rng.uniform(0.005, 0.2))
    dt = (-rng.uniform(0.0, 0.1, n_c)).astype(np.float32)
    f = (rng.random(n_c) * eps).astype(np.float32)
    return n_c, N, x, v, step, m, eps, dt, f


@pytest.mark.parametrize("seed", range(48))
def test_gate_random(seed):
    n_c, N, x, v, step, m, eps, dt, f = _gate_case(seed)
    ref = O.gate_step(x, v, dt, step, m, eps, f)
    got = gate_gpu(x, v, dt, step, m, eps, f)
    np.testing.assert_array_equal(got[0].view(np.uint32), ref[0].view(np.uint32))
    lg, lr = got[2], ref[2]
    fin = np.isfinite(lr)
    np.testing.assert_array_equal(np.isfinite(lg), fin)
    np.testing.assert_allclose(lg[fin], lr[fin], rtol=1e-6, atol=0)
    for c in range(n_c):
        margin = abs(float(np.float32(f[c] + lr[c])) - eps) if (step[c] >= m and fin[c]) else 1.0
        if margin < MARGIN:
            continue
        assert got[3][c] == ref[3][c], f"chunk {c}"
        assert got[1][c] == pytest.approx(ref[1][c], rel=1e-6, abs=0), f"chunk {c}"


@pytest.mark.parametrize("seed", range(24))
def test_history_gate_random(seed):
    n_c, N, x, v, step, m, eps, dt, f = _gate_case(100 + seed)
    h_new = (x + 0.01 * v).astype(np.float32)
    ref = O.history_gate_step(x, h_new, step, m, eps, f)
    got = history_gate_gpu(x, h_new, step, m, eps, f)
    np.testing.assert_array_equal(got[0].view(np.uint32), ref[0].view(np.uint32))
    dg, dr = got[2], ref[2]
    fin = np.isfinite(dr)
    np.testing.assert_array_equal(np.isfinite(dg), fin)
    np.testing.assert_allclose(dg[fin], dr[fin], rtol=1e-6, atol=0)
    for c in range(n_c):
        margin = abs(float(np.float32(f[c] + dr[c])) - eps) if (step[c] >= m and fin[c]) else 1.0
        if margin < MARGIN:
            continue
        assert got[3][c] == ref[3][c] and got[1][c] == pytest.approx(ref[1][c], rel=1e-6)


@pytest.mark.parametrize("seed", range(16))
def test_cache_commit_random(seed):
    """One compression of a float32 cache buffer with random sizes: B_budget
    any multiple of C or not, n_clean any count that makes the chunk overflow,
    the buffer rows past the n_clean + C candidates poisoned with NaN (they
    must never be read)."""
    rng = np.random.default_rng(11000 + seed)
    H = int(rng.integers(1, 4))
    d = int(rng.choice([64, 128]))
    C = int(rng.integers(1, 200))
    B = C * int(rng.integers(1, 5)) if seed % 2 == 0 else int(rng.integers(C, 4 * C + 1))
    n = B if seed % 4 < 2 else int(rng.integers(max(B - C + 1, 0), B + 1))
    L = n + C
    Lq = int(rng.integers(1, 300))
    pool = int(rng.choice([1, 3, 7]))
    lam = float(rng.uniform(0.0, 1.0))
    g = torch.Generator().manual_seed(seed)
    kb = torch.full((H, B + C, d), float("nan"))
    vb = torch.full((H, B + C, d), float("nan"))
    kb[:, :L] = torch.randn(H, L, d, generator=g)
    vb[:, :L] = torch.randn(H, L, d, generator=g)
    q = torch.randn(H, Lq, d, generator=g)
    kn = torch.full_like(kb, 5.0).to(DEV)
    vn = torch.full_like(vb, 5.0).to(DEV)
    ws = fc.workspace(fc.fc_kv_cache_workspace_size(fc.FC_F32, H, Lq, B, C, d))
    idx = torch.empty(H, B, dtype=torch.int32, device=DEV)
    n_next, comp = fc.fc_kv_cache_commit(q.to(DEV), kb.to(DEV), vb.to(DEV), kn, vn, n, C, ws,
                                         pool, lam, idx=idx)
    torch.cuda.synchronize()
    assert comp and n_next == B
    kc = f64(kb[:, :L])
    sc_r = O.score(O.importance(f64(q), kc), O.redundancy(kc), lam, pool)
    gi = idx.cpu().numpy()
    assert gi.min() >= 0 and gi.max() < L
    for h in range(H):
        span = max(float(np.abs(sc_r[h]).max()), 1e-30)
        assert_selection_matches(gi[h:h + 1], sc_r[h:h + 1].astype(np.float64), B, TOL_F32 * span)
        sel = torch.from_numpy(gi[h].astype(np.int64))
        assert torch.equal(kn[h, :B].cpu(), kb[h].index_select(0, sel))
        assert torch.equal(vn[h, :B].cpu(), vb[h].index_select(0, sel))
        assert torch.all(kn[h, B:] == 5.0)


@pytest.mark.parametrize("seed", range(8))
def test_cache_commit_random_bf16(seed):
    """The tensor-core path of a compression inside a cache buffer: random
    head dims, chunk sizes that may not divide the budget, a clean count that
    leaves fewer than B_budget + C candidates, the rows past them NaN."""
    rng = np.random.default_rng(12000 + seed)
    H = int(rng.integers(1, 4))
    d = int(rng.choice([64, 128]))
    C = int(rng.integers(100, 700))
    B = int(rng.integers(C, 3 * C))
    n = int(rng.integers(max(B - C + 1, 0), B + 1))
    L = n + C
    Lq = int(rng.integers(1, 400))
    pool = int(rng.choice([1, 3, 7]))
    lam = float(rng.uniform(0.2, 0.8))
    g = torch.Generator().manual_seed(500 + seed)
    kb = torch.full((H, B + C, d), float("nan")).to(torch.bfloat16)
    vb = torch.full((H, B + C, d), float("nan")).to(torch.bfloat16)
    kb[:, :L] = torch.randn(H, L, d, generator=g).to(torch.bfloat16)
    vb[:, :L] = torch.randn(H, L, d, generator=g).to(torch.bfloat16)
    q = torch.randn(H, Lq, d, generator=g).to(torch.bfloat16)
    kn = torch.full_like(kb, 5.0).to(DEV)
    vn = torch.full_like(vb, 5.0).to(DEV)
    ws = fc.workspace(fc.fc_kv_cache_workspace_size(fc.FC_BF16, H, Lq, B, C, d))
    idx = torch.empty(H, B, dtype=torch.int32, device=DEV)
    n_next, comp = fc.fc_kv_cache_commit(q.to(DEV), kb.to(DEV), vb.to(DEV), kn, vn, n, C, ws,
                                         pool, lam, idx=idx)
    torch.cuda.synchronize()
    assert comp and n_next == B
    assert fc.fc_check_workspace(fc.FC_WS_CACHE, ws)
    kc = f64(kb[:, :L])
    sc_r = O.score(O.importance(f64(q), kc), O.redundancy(kc), lam, pool)
    gi = idx.cpu().numpy()
    assert gi.min() >= 0 and gi.max() < L
    for h in range(H):
        span = max(float(sc_r[h].max() - sc_r[h].min()), 1e-30)
        assert_selection_matches(gi[h:h + 1], sc_r[h:h + 1].astype(np.float64), B, TOL_BF16 * span)
        sel = torch.from_numpy(gi[h].astype(np.int64))
        assert torch.equal(kn[h, :B].cpu(), kb[h].index_select(0, sel))
        assert torch.equal(vn[h, :B].cpu(), vb[h].index_select(0, sel))
        assert torch.all(kn[h, B:].float() == 5.0)
