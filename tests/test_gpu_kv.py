"""GPU parity of the KV-compression calls against the CPU oracle.

Importance and redundancy: float32 inputs within 1e-5 relative; bf16 inputs
(float32 accumulation) within 1e-4 relative plus 1e-4 of the head's largest
value.  Score and top-B on identical float32 inputs: bitwise scores and
identical indices (both decide in float32).  Compaction: bitwise.  The whole
chain on the workloads: scores within the stated tolerance of the head's
score range, index sets equal up to the margin waiver."""

import numpy as np
import pytest
import torch

from cache_gating_kv_b200 import workloads as W
from oracle import flowcache_oracle as O
from tests.gpu_util import (TOL_BF16, TOL_F32, assert_selection_matches, compact_gpu, f64,
                            importance_gpu, redundancy_gpu, score_topb_gpu)

pytestmark = pytest.mark.gpu


def _close(got, ref, bf16):
    if bf16:
        atol = 1e-4 * np.abs(ref).max(axis=-1, keepdims=True)
        assert np.all(np.abs(got - ref) <= 1e-4 * np.abs(ref) + atol), \
            float(np.max(np.abs(got - ref) / (np.abs(ref) + atol)))
    else:
        np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-9 * np.abs(ref).max())


def _rand_qk(H, Lq, Lk, d, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(H, Lq, d, generator=g).to(dtype)
    k = torch.randn(H, Lk, d, generator=g).to(dtype)
    return q, k


# ---------------------------------------------------------------------------
# importance
# ---------------------------------------------------------------------------
def test_importance_tiny_fp32_full():
    cfg = W.KV_CONFIGS["tiny_fp32"]
    q, k, _ = W.kv_inputs(cfg, seed=0)
    got = importance_gpu(q, k)
    ref = O.importance(f64(q), f64(k))
    _close(got, ref, bf16=False)
    np.testing.assert_allclose(got.sum(axis=1), 1.0, rtol=1e-5)


@pytest.mark.parametrize("H,Lq,Lk,d,dtype", [
    (3, 300, 777, 128, torch.bfloat16), (2, 129, 1000, 64, torch.bfloat16),
    (1, 1, 5, 128, torch.bfloat16), (2, 257, 130, 64, torch.float32),
    (1, 64, 64, 128, torch.float32), (2, 1000, 385, 128, torch.bfloat16),
    # 306 key tiles of 128 (the last of each head partial): 148 two-tile CTAs
    # and 10 one-tile CTAs in the column pass
    (3, 300, 13000, 128, torch.bfloat16)])
def test_importance_ragged(H, Lq, Lk, d, dtype):
    q, k = _rand_qk(H, Lq, Lk, d, dtype, seed=Lq + Lk)
    got = importance_gpu(q, k)
    _close(got, O.importance(f64(q), f64(k)), bf16=dtype == torch.bfloat16)


def test_importance_explicit_scale_and_sharp_softmax():
    q, k = _rand_qk(2, 200, 500, 128, torch.bfloat16, seed=5)
    got = importance_gpu(q, k, scale=0.5)  # ~5.7x the default: a peaked softmax
    _close(got, O.importance(f64(q), f64(k), scale=0.5), bf16=True)


@pytest.mark.parametrize("d,dtype,grow", [(128, torch.bfloat16, 1), (64, torch.bfloat16, 1),
                                           (128, torch.bfloat16, -1), (128, torch.float32, 1)])
def test_importance_logits_drifting_along_keys(d, dtype, grow):
    """Keys drift towards (grow=1) or away from (grow=-1) the queries' common
    direction, so along a row the logits rise (or fall) by ~200 in log2 units
    from the first key to the last, ~15 within every 128-key slice that one
    epilogue warp drains: the row pass must move its reference again and
    again, inside slices too (its rare overflow path), and the column pass
    must still weigh every query by the right normaliser."""
    g = torch.Generator().manual_seed(11 + d)
    H, Lq, Lk = 2, 300, 1700
    u = torch.randn(H, 1, d, generator=g)
    u = u / u.norm(dim=-1, keepdim=True)
    q = torch.randn(H, Lq, d, generator=g) * 0.3 + 3.0 * u
    c = np.log2(np.e) / np.sqrt(d)
    amp = 200.0 / (3.0 * c)  # q.k grows by ~3 * amp along the row
    ramp = torch.linspace(0.0, 1.0, Lk) if grow > 0 else torch.linspace(1.0, 0.0, Lk)
    k = torch.randn(H, Lk, d, generator=g) + (amp * ramp)[None, :, None] * u
    q, k = q.to(dtype), k.to(dtype)
    got = importance_gpu(q, k)
    ref = O.importance(f64(q), f64(k))
    assert np.all(np.isfinite(got))
    _close(got, ref, bf16=dtype == torch.bfloat16)
    np.testing.assert_allclose(got.sum(axis=1), 1.0, rtol=1e-4)


@pytest.mark.parametrize("name", ["bf16_layer", "bf16_large_head"])
def test_importance_workload_sampled_heads(name):
    """All heads go through the kernel; two heads are checked against the
    oracle in full (row normalisers + every column)."""
    cfg = W.KV_CONFIGS[name]
    q, k, _ = W.kv_inputs(cfg, seed=0)
    got = importance_gpu(q, k)
    np.testing.assert_allclose(got.sum(axis=1), 1.0, rtol=2e-4)
    for h in (0, cfg.H - 1):
        ref = O.importance(f64(q[h:h + 1]), f64(k[h:h + 1]))
        _close(got[h:h + 1], ref, bf16=True)


# ---------------------------------------------------------------------------
# redundancy
# ---------------------------------------------------------------------------
def test_redundancy_tiny_fp32_full():
    cfg = W.KV_CONFIGS["tiny_fp32"]
    _, k, _ = W.kv_inputs(cfg, seed=0)
    got = redundancy_gpu(k)
    _close(got, O.redundancy(f64(k)), bf16=False)


@pytest.mark.parametrize("H,Lk,d,dtype", [
    (3, 777, 128, torch.bfloat16), (2, 1, 64, torch.bfloat16), (2, 5000, 64, torch.float32),
    (1, 33, 128, torch.float32), (4, 4099, 128, torch.bfloat16)])
def test_redundancy_ragged(H, Lk, d, dtype):
    _, k = _rand_qk(H, 1, Lk, d, dtype, seed=Lk)
    _close(redundancy_gpu(k), O.redundancy(f64(k)), bf16=False)


def test_redundancy_degenerate_keys():
    k = torch.randn(3, 300, 128).to(torch.bfloat16)
    k[0, 17] = 0  # zero key: r = 0
    k[1] = k[1, :1].expand(300, 128)  # all identical: uniform
    k[2, 10:20] = k[2, 50]  # duplicates raise redundancy
    got = redundancy_gpu(k)
    _close(got, O.redundancy(f64(k)), bf16=False)
    np.testing.assert_allclose(got[1], 1 / 300, rtol=1e-6)


@pytest.mark.parametrize("name", ["bf16_layer", "long_history"])
def test_redundancy_workload_sampled(name):
    """Every head through the kernel; sampled columns of two heads against the
    oracle's brute-force logits r_j, through log(Red_j / Red_0) = r_j - r_0."""
    cfg = W.KV_CONFIGS[name]
    heads = list(range(cfg.H)) if name != "long_history" else [0, 1, 2, 3]
    _, k, _ = W.kv_inputs(cfg, seed=0, heads=heads)
    got = redundancy_gpu(k)
    np.testing.assert_allclose(got.sum(axis=1), 1.0, rtol=1e-5)
    rng = np.random.default_rng(0)
    for h in (0, len(heads) - 1):
        cols = np.concatenate([[0], rng.choice(k.shape[1], 40, replace=False)])
        r = O.redundancy_logits_at(f64(k), [h] * cols.size, cols)
        lr = np.log(got[h, cols].astype(np.float64))
        np.testing.assert_allclose(lr - lr[0], r - r[0], atol=2e-6)


# ---------------------------------------------------------------------------
# score + top-B (same float32 inputs on both sides: exact)
# ---------------------------------------------------------------------------
def _synthetic_imp_red(H, Lk, seed, dup_frac=0.0):
    rng = np.random.default_rng(seed)
    g = rng.gamma(0.5, size=(H, Lk))
    imp = (g / g.sum(axis=1, keepdims=True)).astype(np.float32)
    e = rng.uniform(0.9, 1.1, size=(H, Lk))
    if dup_frac:
        n = int(Lk * dup_frac)
        for h in range(H):
            pos = rng.choice(Lk, n, replace=False)
            e[h, pos] = e[h, rng.integers(0, Lk, n)]
            imp[h, pos[: n // 2]] = imp[h, pos[n // 2: n // 2 * 2]]
    red = (e / e.sum(axis=1, keepdims=True)).astype(np.float32)
    return imp, red


@pytest.mark.parametrize("H,Lk,B,pool,lam", [
    (2, 1024, 256, 7, 0.5), (3, 1000, 1, 7, 0.5), (3, 1000, 999, 3, 0.3), (1, 1, 1, 7, 0.5),
    (2, 777, 300, 1, 0.7), (2, 5000, 2500, 511, 0.5), (4, 16384, 8192, 7, 0.5),
    (2, 3000, 1000, 7, 1.0), (2, 3000, 1000, 7, 0.0), (2, 3000, 1000, 7, -0.25)])
def test_score_topb_exact(H, Lk, B, pool, lam):
    imp, red = _synthetic_imp_red(H, Lk, seed=Lk + B, dup_frac=0.25)
    sc_ref, idx_ref = O.score_topb(imp, red, lam, pool, B)
    sc, idx = score_topb_gpu(imp, red, pool, lam, B)
    np.testing.assert_array_equal(sc.view(np.uint32), sc_ref.view(np.uint32))
    np.testing.assert_array_equal(idx, idx_ref)


@pytest.mark.parametrize("Lk,B", [(10, 10), (10, 25), (1, 4)])
def test_score_topb_keep_all(Lk, B):
    imp, red = _synthetic_imp_red(2, Lk, seed=1)
    _, idx = score_topb_gpu(imp, red, 7, 0.5, B, want_score=False)
    np.testing.assert_array_equal(idx, O.topb(O.score(imp, red, 0.5, 7), B))


def test_score_topb_ties_and_signed_zero():
    H, Lk = 3, 4096
    imp = np.zeros((H, Lk), np.float32)
    red = np.zeros((H, Lk), np.float32)
    red[1, ::3] = 1e-3  # a third of head 1 loses; the rest ties at 0
    imp[2, 100] = 1.0  # head 2: pooled importance plateau around 100
    for lam in (0.5, -0.5):  # lam < 0 gives -0 scores that must tie with +0
        sc_ref, idx_ref = O.score_topb(imp, red, lam, 7, 1500)
        sc, idx = score_topb_gpu(imp, red, 7, lam, 1500)
        np.testing.assert_array_equal(idx, idx_ref)
        np.testing.assert_array_equal(sc.view(np.uint32), sc_ref.view(np.uint32))


@pytest.mark.parametrize("Lk", [65536, 131072, 196608])
def test_score_topb_long_heads_mass_ties(Lk):
    """Long heads (one 16-CTA cluster per head, the keys written over the
    pooling tile) where most scores are equal: far more keys than the
    candidate buffer holds share the threshold's top 16 bits, so the last two
    radix passes scan the whole slice; the threshold falls inside the tie."""
    H, B = 3, Lk // 4
    rng = np.random.default_rng(Lk)
    imp = np.full((H, Lk), 1.0 / Lk, np.float32)
    red = np.full((H, Lk), 1.0 / Lk, np.float32)
    imp[0, rng.choice(Lk, Lk // 16, replace=False)] = 2.0 / Lk  # pooled: ~40% above the tie
    red[1, rng.choice(Lk, Lk // 2, replace=False)] = 0.5 / Lk   # half above, half tied
    # head 2: every score ties; the B lowest indices are kept
    sc_ref, idx_ref = O.score_topb(imp, red, 0.5, 7, B)
    sc, idx = score_topb_gpu(imp, red, 7, 0.5, B)
    np.testing.assert_array_equal(sc.view(np.uint32), sc_ref.view(np.uint32))
    np.testing.assert_array_equal(idx, idx_ref)
    np.testing.assert_array_equal(idx[2], np.arange(B, dtype=np.int32))


@pytest.mark.parametrize("Lk,B", [(131072, 32768), (65536, 16384), (32760, 16380)])
def test_score_topb_full_size_exact(Lk, B):
    """Full per-layer sizes (40 heads), including the case whose keys do not
    fit in shared memory; 25% duplicated values make exact ties."""
    imp, red = _synthetic_imp_red(40, Lk, seed=Lk, dup_frac=0.25)
    sc_ref, idx_ref = O.score_topb(imp, red, 0.5, 7, B)
    sc, idx = score_topb_gpu(imp, red, 7, 0.5, B)
    np.testing.assert_array_equal(sc.view(np.uint32), sc_ref.view(np.uint32))
    np.testing.assert_array_equal(idx, idx_ref)


def test_score_topb_deterministic():
    imp, red = _synthetic_imp_red(8, 20000, seed=3, dup_frac=0.25)
    a = score_topb_gpu(imp, red, 7, 0.5, 5000)
    b = score_topb_gpu(imp, red, 7, 0.5, 5000)
    np.testing.assert_array_equal(a[1], b[1])
    np.testing.assert_array_equal(a[0].view(np.uint32), b[0].view(np.uint32))


# ---------------------------------------------------------------------------
# compaction (bitwise)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("H,Lk,d,B,dtype", [
    (3, 1000, 128, 300, torch.bfloat16), (2, 77, 64, 77, torch.bfloat16),
    (2, 500, 128, 257, torch.float32), (1, 9, 64, 3, torch.float32),
    (24, 16384, 128, 8192, torch.bfloat16)])
def test_compact_bitwise(H, Lk, d, B, dtype):
    g = torch.Generator().manual_seed(B)
    k = torch.randn(H, Lk, d, generator=g).to(dtype)
    v = torch.randn(H, Lk, d, generator=g).to(dtype)
    rng = np.random.default_rng(B)
    idx = np.stack([np.sort(rng.choice(Lk, B, replace=False)) for _ in range(H)]).astype(np.int32)
    idx[0, -1] = -1  # padding row -> zeros
    ko, vo = compact_gpu(k, v, idx)
    kr, vr = O.compact(k.float().numpy(), v.float().numpy(), idx)
    np.testing.assert_array_equal(ko.float().numpy(), kr)
    np.testing.assert_array_equal(vo.float().numpy(), vr)


# ---------------------------------------------------------------------------
# the whole compression chain on the workloads
# ---------------------------------------------------------------------------
def _chain(q, k, v, cfg, lam, B):
    imp = importance_gpu(q, k)
    red = redundancy_gpu(k)
    sc, idx = score_topb_gpu(imp, red, cfg.pool, lam, B)
    ko, vo = compact_gpu(k, v, idx)
    return imp, red, sc, idx, ko, vo


@pytest.mark.parametrize("name,heads", [("tiny_fp32", None), ("bf16_layer", [0, 23]),
                                        ("bf16_large_head", [5])])
def test_compression_chain_against_oracle(name, heads):
    cfg = W.KV_CONFIGS[name]
    q, k, v = W.kv_inputs(cfg, seed=0)
    bf16 = cfg.dtype == "bf16"
    tol = TOL_BF16 if bf16 else TOL_F32
    heads = list(range(cfg.H)) if heads is None else heads
    for lam in cfg.lam:
        imp, red, sc, idx, ko, vo = _chain(q, k, v, cfg, lam, cfg.B)
        for h in heads:
            imp_r = O.importance(f64(q[h:h + 1]), f64(k[h:h + 1]))
            red_r = O.redundancy(f64(k[h:h + 1]))
            sc_r, _ = O.score_topb(imp_r, red_r, lam, cfg.pool, cfg.B)
            span = (sc_r.max() - sc_r.min()) if bf16 else np.abs(sc_r).max()
            assert np.max(np.abs(sc[h] - sc_r[0])) <= tol * span
            assert_selection_matches(idx[h:h + 1], sc_r.astype(np.float64), cfg.B, tol * span)
        # the chain's compaction holds exactly the rows its selection names
        sel = torch.from_numpy(idx.astype(np.int64))
        for h in heads:
            assert torch.equal(ko[h], k[h].index_select(0, sel[h]))
            assert torch.equal(vo[h], v[h].index_select(0, sel[h]))


@pytest.mark.parametrize("d,dtype", [(64, torch.float32), (128, torch.float32),
                                     (64, torch.bfloat16), (128, torch.bfloat16)])
def test_redundancy_long_heads_sampled(d, dtype):
    """L_k >= 65536 takes the four-rows-in-flight variant: rows sum to one and
    sampled log-ratios match the oracle's brute-force logits."""
    H, Lk = 2, 70001
    g = torch.Generator().manual_seed(d)
    k = (torch.randn(H, Lk, d, generator=g) + 0.3 * torch.randn(H, 1, d, generator=g)).to(dtype)
    red = redundancy_gpu(k)
    np.testing.assert_allclose(red.sum(axis=1), 1.0, rtol=1e-5)
    rng = np.random.default_rng(d)
    for h in range(H):
        cols = np.sort(rng.choice(Lk, 24, replace=False))
        r = O.redundancy_logits_at(f64(k[h:h + 1]), [0] * cols.size, cols)
        lr = np.log(red[h, cols].astype(np.float64))
        np.testing.assert_allclose(lr - lr[0], r - r[0], atol=2e-6)
