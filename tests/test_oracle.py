"""Pins for the CPU oracle: every check here is fixed by the pages' definitions,
by mathematics (closed forms, invariants, brute force) or by an independent
library routine -- never by the oracle itself and never by the CUDA path.

Definitions: "Flow Caching for Autoregressive Video Generation" (papernotes.org),
方法详解 / 关键设计 1 (relative L1), 关键设计 2 (accumulator f), 关键设计 3
(importance / redundancy / score / top-B / compaction).
"""

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import flowcache_oracle as O


# ---------------------------------------------------------------------------
# Gate: key designs 1 and 2
# ---------------------------------------------------------------------------
def test_gate_hand_trace_constant(golden_dir):
    """Hand-worked mask / f sequence with exactly representable numbers."""
    g = json.load(open(os.path.join(golden_dir, "gate_trace_constant.json")))
    N = g["N"]
    f = np.zeros(1, np.float32)
    for t in range(g["steps"]):
        x = np.full((1, N), g["x"], np.float32)  # reset X before every step
        v = np.full((1, N), g["v"], np.float32)
        x_next, f, l1, mask = O.gate_step(x, v, np.float32([g["dt"]]), np.int32([t]),
                                          g["m"], g["eps"], f)
        assert l1[0] == np.float32(g["l1"][t])
        assert mask[0] == g["mask"][t], t
        assert f[0] == np.float32(g["f"][t]), t
        assert np.all(x_next == np.float32(g["x_next"]))


def test_gate_evolving_latent_denominator_is_pre_update():
    """X evolves: X_k = 1 - k/64 (exact).  L1 at step k = (1/64)/(1 - k/64)
    = 1/(64-k): the denominator is ||X_t||_1 before the update."""
    N = 512
    x = np.ones((1, N), np.float32)
    v = np.full((1, N), 0.5, np.float32)
    dt = np.float32([-1.0 / 32.0])  # v*dt = -1/64 exactly
    f = np.zeros(1, np.float32)
    for k in range(20):
        x_next, f, l1, mask = O.gate_step(x, v, dt, np.int32([k]), 1000, 1.0, f)
        assert l1[0] == np.float32(1.0 / (64 - k))
        assert np.all(x_next == np.float32(1.0 - (k + 1) / 64.0))
        assert mask[0] == 1 and f[0] == 0.0  # k < m: forced
        x = x_next


def test_gate_signs_and_abs():
    """Mixed-sign latents and velocities: both norms take absolute values."""
    N = 256
    x = np.where(np.arange(N) % 2 == 0, 2.0, -2.0).astype(np.float32)[None]
    v = np.where(np.arange(N) % 3 == 0, -1.0, 1.0).astype(np.float32)[None]
    x_next, _, l1, _ = O.gate_step(x, v, np.float32([0.25]), np.int32([0]), 0, 10.0,
                                   np.zeros(1, np.float32))
    assert l1[0] == np.float32(0.125)  # (N*0.25)/(N*2)
    assert np.all(x_next == x + v * np.float32(0.25))


def test_gate_corollary1_heterogeneous_norms():
    """Corollary 1: the same update on chunks of different ||X||_1 gives
    different L1 (here exactly in the inverse ratio of the norms)."""
    N = 1024
    x = np.stack([np.full(N, 1.0, np.float32), np.full(N, 2.0, np.float32)])
    v = np.full((2, N), 0.75, np.float32)
    _, _, l1, _ = O.gate_step(x, v, np.float32([0.125, 0.125]), np.int32([3, 3]), 0, 1.0,
                              np.zeros(2, np.float32))
    assert l1[0] != l1[1]
    assert l1[0] == np.float32(2.0) * l1[1]


def test_gate_inactive_untouched_and_zero_norm():
    N = 64
    x = np.stack([np.ones(N), np.zeros(N), np.zeros(N), np.ones(N)]).astype(np.float32)
    v = np.stack([np.ones(N), np.ones(N), np.zeros(N), np.ones(N)]).astype(np.float32)
    f0 = np.float32([0.5, 0.0, 0.0, 0.25])
    x_next, f, l1, mask = O.gate_step(x, v, np.float32([0.5, 0.5, 0.5, 0.5]),
                                      np.int32([-1, 7, 7, 7]), 2, 100.0, f0)
    # inactive chunk 0: nothing changes
    assert np.all(x_next[0] == x[0]) and f[0] == f0[0] and l1[0] == 0 and mask[0] == 0
    # ||X||_1 = 0 with a non-zero update: L1 = +inf -> recompute
    assert np.isinf(l1[1]) and mask[1] == 1 and f[1] == 0
    # ||X||_1 = 0 and a zero update: L1 = 0 -> reuse
    assert l1[2] == 0 and mask[2] == 0 and f[2] == 0
    # an ordinary chunk: L1 = 0.5, f = 0.25 + 0.5 = 0.75 <= 100 -> reuse
    assert l1[3] == np.float32(0.5) and mask[3] == 0 and f[3] == np.float32(0.75)


def test_gate_strict_threshold():
    """Key design 2 compares with '> eps': equality reuses."""
    N = 1024
    x = np.ones((1, N), np.float32)
    v = np.ones((1, N), np.float32)
    dt = np.float32([-1.0 / 64])
    for f_prev, eps, expect in [(0.03125, 0.046875, 0), (0.03125, 0.0468749, 1)]:
        _, f, _, mask = O.gate_step(x, v, dt, np.int32([5]), 2, eps, np.float32([f_prev]))
        assert mask[0] == expect
        assert f[0] == (np.float32(0.046875) if expect == 0 else 0.0)


def test_gate_forced_steps_count_per_chunk():
    """'first m steps' counts per chunk: chunk with step < m is forced even if
    its L1 is tiny; chunk with step >= m follows the accumulator."""
    N = 128
    x = np.ones((2, N), np.float32)
    v = np.full((2, N), 1e-3, np.float32)
    _, f, _, mask = O.gate_step(x, v, np.float32([1.0, 1.0]), np.int32([4, 5]), 5, 0.5,
                                np.float32([0.2, 0.2]))
    assert list(mask) == [1, 0]
    assert f[0] == 0.0 and f[1] > np.float32(0.2)


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_gate_theorem1_monotone_on_flow_matching_toy(seed):
    """Theorem 1: at the exact flow-matching velocity with sigma(t) = (t/T)^p,
    L1_rel rises monotonically along the trajectory.  Toy: single-point data
    x0 (std 0.1), x_s = s*x0 + (1-s)*noise, exact velocity x0 - noise, Euler
    steps dt = sigma(t+1) - sigma(t), p = 2, T = 30.  The pages do not print the
    theorem's assumptions; the rise is regime dependent (a large x0, or p <= 1,
    breaks it), and this is a regime where it holds."""
    rng = np.random.default_rng(100 + seed)
    N, T, p = 16384, 30, 2.0
    x0 = rng.standard_normal(N) * 0.1
    noise = rng.standard_normal(N)
    x = noise.astype(np.float32)[None]
    v = (x0 - noise).astype(np.float32)[None]
    f = np.zeros(1, np.float32)
    l1s = []
    for t in range(T - 1):
        dt = np.float32([((t + 1) / T) ** p - (t / T) ** p])
        x, f, l1, _ = O.gate_step(x, v, dt, np.int32([t]), 0, 1e9, f)
        l1s.append(float(l1[0]))
    assert all(b > a for a, b in zip(l1s, l1s[1:]))


# ---------------------------------------------------------------------------
# Importance: key design 3
# ---------------------------------------------------------------------------
def _worked(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "kv_worked_example.json")))
    k = np.array(g["keys"], np.float64)[None]
    q = np.array([[math.sqrt(2) * math.log(2), 0.0], [0.0, math.sqrt(2) * math.log(3)]])[None]
    return g, q, k


def test_importance_worked_example(golden_dir):
    g, q, k = _worked(golden_dir)
    exp = np.array([(float(Fraction(a)) + float(Fraction(b))) / 2
                    for a, b in g["importance_rational"]])
    imp = O.importance(q, k)
    np.testing.assert_allclose(imp[0], exp, rtol=0, atol=1e-14)


def test_importance_sums_to_one_and_single_query_is_softmax():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((3, 37, 16))
    k = rng.standard_normal((3, 301, 16))
    imp = O.importance(q, k)
    np.testing.assert_allclose(imp.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    # L_q = 1: a single softmax row (library routine, torch fp64)
    imp1 = O.importance(q[:, :1], k)
    ref = torch.softmax(torch.from_numpy(q[:, :1]) @ torch.from_numpy(k).transpose(1, 2)
                        / 4.0, dim=-1)[:, 0].numpy()
    np.testing.assert_allclose(imp1, ref, rtol=1e-12, atol=1e-15)


def test_importance_matches_library_attention_weights():
    """Mean over queries of the attention weights returned by torch's
    scaled_dot_product_attention with V = identity (so O = P)."""
    rng = np.random.default_rng(1)
    H, Lq, Lk, d = 2, 19, 53, 8
    q = rng.standard_normal((H, Lq, d))
    k = rng.standard_normal((H, Lk, d)) * 2.0
    eye = torch.eye(Lk, dtype=torch.float64).expand(H, Lk, Lk)
    P = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), eye)
    np.testing.assert_allclose(O.importance(q, k), P.mean(dim=1).numpy(), rtol=1e-11, atol=1e-15)
    # an explicit scale is honoured (here twice the default)
    P2 = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), eye, scale=2.0 / math.sqrt(d))
    np.testing.assert_allclose(O.importance(q, k, scale=2.0 / math.sqrt(d)),
                               P2.mean(dim=1).numpy(), rtol=1e-11, atol=1e-15)


def test_importance_two_keys_closed_form():
    """Two keys: Imp_1 = mean_q logistic(q.(k1-k2)/sqrt(d))."""
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 50, 4))
    k = rng.standard_normal((1, 2, 4))
    z = (q[0] @ (k[0, 0] - k[0, 1])) / 2.0
    np.testing.assert_allclose(O.importance(q, k)[0, 0], np.mean(1 / (1 + np.exp(-z))),
                               rtol=1e-13)


def test_importance_degenerate_cases():
    rng = np.random.default_rng(3)
    k = rng.standard_normal((1, 40, 8))
    np.testing.assert_allclose(O.importance(np.zeros((1, 5, 8)), k), 1 / 40, rtol=1e-14)
    k[0, 7] = k[0, 21]
    imp = O.importance(rng.standard_normal((1, 9, 8)), k)
    assert imp[0, 7] == imp[0, 21]


def test_row_lse_and_sampled_importance_agree_with_full():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((2, 300, 16))
    k = rng.standard_normal((2, 700, 16))
    lse = O.row_lse(q, k)
    ref = torch.logsumexp(torch.from_numpy(q) @ torch.from_numpy(k).transpose(1, 2) / 4.0,
                          dim=-1).numpy()
    np.testing.assert_allclose(lse, ref, rtol=1e-13)
    full = O.importance(q, k)
    heads, cols = [0, 1, 1, 0], [0, 5, 699, 350]
    np.testing.assert_allclose(O.importance_at(q, k, heads, cols, lse),
                               full[heads, cols], rtol=1e-11)


# ---------------------------------------------------------------------------
# Redundancy: key design 3
# ---------------------------------------------------------------------------
def test_redundancy_worked_example(golden_dir):
    g, _, k = _worked(golden_dir)
    s = 1 / math.sqrt(2)
    r = np.array([(1 + s) / 4, (1 + s) / 4, s / 4, 3 * s / 4])
    exp = np.exp(r) / np.exp(r).sum()
    np.testing.assert_allclose(O.redundancy(k)[0], exp, rtol=1e-14)


def test_redundancy_two_direction_closed_form():
    """n1 keys along a, n2 along b (random magnitudes), cos(a,b) = c:
    r = ((n1-1) + n2*c)/L for group 1 and ((n2-1) + n1*c)/L for group 2.
    Pins the zeroed diagonal, the 1/L_k, the normalisation and the softmax."""
    rng = np.random.default_rng(5)
    d, n1, n2 = 6, 9, 4
    a = rng.standard_normal(d); a /= np.linalg.norm(a)
    b = rng.standard_normal(d); b /= np.linalg.norm(b)
    c = a @ b
    keys = [a * m for m in rng.uniform(0.1, 5, n1)] + [b * m for m in rng.uniform(0.1, 5, n2)]
    order = rng.permutation(n1 + n2)
    k = np.array(keys)[order][None]
    L = n1 + n2
    r_grp = np.array([((n1 - 1) + n2 * c) / L] * n1 + [((n2 - 1) + n1 * c) / L] * n2)[order]
    exp = np.exp(r_grp) / np.exp(r_grp).sum()
    np.testing.assert_allclose(O.redundancy(k)[0], exp, rtol=1e-13)


def test_redundancy_invariants():
    rng = np.random.default_rng(6)
    k = rng.standard_normal((2, 200, 16))
    red = O.redundancy(k)
    np.testing.assert_allclose(red.sum(axis=1), 1.0, atol=1e-12)
    # bound from r in [-1, 1]: e^-2/L <= Red <= e^2/L
    assert np.all(red >= math.exp(-2) / 200) and np.all(red <= math.exp(2) / 200)
    # orthogonal keys of different lengths: every r = 0 -> uniform
    ortho = (np.eye(8) * np.arange(1, 9)[:, None])[None]
    np.testing.assert_allclose(O.redundancy(ortho), 1 / 8, rtol=1e-14)
    # duplicating a key raises its redundancy and its twin's
    k2 = k[:1].copy()
    base = O.redundancy(k2)[0]
    k2[0, 50] = k2[0, 120]
    dup = O.redundancy(k2)[0]
    assert dup[50] > base[50] and dup[120] > base[120]
    assert dup[50] == pytest.approx(dup[120], rel=1e-12)
    # a zero key normalises to zero: r_zero = 0
    k3 = k[:1].copy()
    k3[0, 3] = 0.0
    r = O.redundancy_logits_at(k3, [0], [3])
    assert r[0] == 0.0


def test_redundancy_equals_sum_identity():
    """Independent route: sum_{i != j} khat_i.khat_j = khat_j.(sum_i khat_i)
    - ||khat_j||^2.  Must match the brute-force matrix to 1e-12."""
    rng = np.random.default_rng(7)
    k = rng.standard_normal((2, 300, 24))
    k[1, 10] = 0.0
    kt = torch.from_numpy(k)
    kh = torch.nn.functional.normalize(kt, dim=-1, eps=1e-12)
    s = kh.sum(dim=1, keepdim=True)
    r = ((kh * s).sum(-1) - (kh * kh).sum(-1)) / k.shape[1]
    ref = torch.softmax(r, dim=-1).numpy()
    np.testing.assert_allclose(O.redundancy(k), ref, rtol=1e-12)
    heads, cols = [0, 1, 1], [0, 10, 299]
    np.testing.assert_allclose(O.redundancy_logits_at(k, heads, cols),
                               r.numpy()[heads, cols], atol=1e-14)


# ---------------------------------------------------------------------------
# Pooling, score, top-B, compaction: key design 3
# ---------------------------------------------------------------------------
def test_maxpool_matches_library():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((3, 101))
    ref = torch.nn.functional.max_pool1d(torch.from_numpy(x)[:, None], 7, 1, 3)[:, 0].numpy()
    np.testing.assert_array_equal(O.maxpool1d(x, 7), ref)
    ref3 = torch.nn.functional.max_pool1d(torch.from_numpy(x)[:, None], 3, 1, 1)[:, 0].numpy()
    np.testing.assert_array_equal(O.maxpool1d(x, 3), ref3)
    np.testing.assert_array_equal(O.maxpool1d(x, 1), x)


def test_score_float32_definition():
    """lam = 1/2 scales by a power of two: fl(fl(p/2) - fl(r/2)) = fl(p - r)/2."""
    rng = np.random.default_rng(9)
    imp = rng.random((2, 64)).astype(np.float32)
    red = rng.random((2, 64)).astype(np.float32)
    sc = O.score(imp, red, 0.5, 5)
    pooled = torch.nn.functional.max_pool1d(torch.from_numpy(imp)[:, None], 5, 1, 2)[:, 0].numpy()
    np.testing.assert_array_equal(sc, (pooled - red) * np.float32(0.5))
    assert sc.dtype == np.float32


def test_topb_lambda_extremes_against_library():
    rng = np.random.default_rng(10)
    imp = rng.random((3, 500)).astype(np.float32)
    red = rng.random((3, 500)).astype(np.float32)
    B = 77
    _, idx1 = O.score_topb(imp, red, 1.0, 7, B)  # pure importance (LLM-style)
    pooled = torch.nn.functional.max_pool1d(torch.from_numpy(imp)[:, None], 7, 1, 3)[:, 0]
    _, idx0 = O.score_topb(imp, red, 0.0, 7, B)  # least redundant
    ref0 = torch.topk(-torch.from_numpy(red), B, dim=1).indices.sort(dim=1).values.numpy()
    np.testing.assert_array_equal(idx0, ref0)
    # pooled importance has plateaus (ties); the kept set must contain every
    # token strictly above the B-th value and be filled lowest-index-first
    for h in range(3):
        p = pooled[h].numpy()
        thr = np.sort(p)[::-1][B - 1]
        above = np.flatnonzero(p > thr)
        ties = np.flatnonzero(p == thr)
        exp = np.sort(np.concatenate([above, ties[:B - above.size]]))
        np.testing.assert_array_equal(idx1[h], exp)


def test_topb_brute_force_enumeration():
    """Tiny heads with integer-valued scores (many ties): the kept set is the
    subset of size B with the largest score sum, and among those the one that
    keeps the lowest indices (lexicographically smallest sorted tuple)."""
    rng = np.random.default_rng(11)
    for trial in range(40):
        L = int(rng.integers(1, 11))
        B = int(rng.integers(1, L + 1))
        sc = rng.integers(-3, 4, size=(1, L)).astype(np.float32)
        best = None
        for sub in itertools.combinations(range(L), B):
            key = (-sum(sc[0, list(sub)]), sub)
            if best is None or key < best:
                best = key
        np.testing.assert_array_equal(O.topb(sc, B)[0], np.array(best[1]))


def test_topb_ties_and_padding():
    sc = np.zeros((2, 10), np.float32)
    np.testing.assert_array_equal(O.topb(sc, 4), [[0, 1, 2, 3]] * 2)
    sc[1, 9] = np.float32(-0.0)  # -0 ties with +0
    np.testing.assert_array_equal(O.topb(sc, 10)[1], np.arange(10))
    np.testing.assert_array_equal(O.topb(sc[:, :3], 5), [[0, 1, 2, -1, -1]] * 2)


def test_compact_is_a_gather():
    rng = np.random.default_rng(12)
    k = rng.standard_normal((2, 30, 4)).astype(np.float32)
    v = rng.standard_normal((2, 30, 4)).astype(np.float32)
    idx = np.array([[0, 5, 29, -1], [1, 2, 3, 4]], np.int32)
    ko, vo = O.compact(k, v, idx)
    kt = torch.from_numpy(k)
    for h in range(2):
        sel = torch.from_numpy(idx[h].clip(min=0)).long()
        np.testing.assert_array_equal(ko[h][idx[h] >= 0], kt[h].index_select(0, sel)[idx[h] >= 0])
    assert np.all(ko[0, 3] == 0) and np.all(vo[0, 3] == 0)
    np.testing.assert_array_equal(vo[1], v[1, 1:5])


# ---------------------------------------------------------------------------
# History-guided gate (the neighbouring ARCache method's HGC rule)
# ---------------------------------------------------------------------------
def test_history_gate_hand_trace(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "history_gate_trace.json")))
    N = g["N"]
    f = np.zeros(1, np.float32)
    for t in range(g["steps"]):
        h_old = np.full((1, N), g["h_old"], np.float32)
        h_new = np.full((1, N), g["h_new"], np.float32)
        h_next, f, d, mask = O.history_gate_step(h_old, h_new, np.int32([t]), g["m"], g["delta"], f)
        assert d[0] == np.float32(g["d"])
        assert mask[0] == g["mask"][t], t
        assert f[0] == np.float32(g["f"][t]), t
        assert np.all(h_next == np.float32(g["h_new"]))


def test_history_gate_denominator_is_the_older_step():
    """h_old = 2, h_new = 3: Delta = 1/2 (older step in the denominator), not 1/3."""
    h_old = np.full((1, 64), 2.0, np.float32)
    h_new = np.full((1, 64), 3.0, np.float32)
    _, _, d, _ = O.history_gate_step(h_old, h_new, np.int32([5]), 0, 10.0, np.zeros(1, np.float32))
    assert d[0] == np.float32(0.5)


def test_history_gate_matches_cumulative_rule_brute_force():
    """Random Delta sequences: the refresh steps are exactly those where the
    window sum from the last refresh (inclusive) first exceeds delta."""
    rng = np.random.default_rng(13)
    for trial in range(20):
        deltas = rng.uniform(0.0, 0.04, size=25).astype(np.float32)
        thr = float(rng.uniform(0.02, 0.1))
        f = np.zeros(1, np.float32)
        got = []
        for t, dv in enumerate(deltas):
            h_old = np.ones((1, 256), np.float32)
            h_new = h_old + np.float32(dv)
            # the Delta the gate sees is the float32 value of (h_new - 1) on each element
            _, f, d, mask = O.history_gate_step(h_old, h_new, np.int32([t]), 0, thr, f)
            got.append((int(mask[0]), float(d[0])))
        # brute force on the observed Deltas: window sums from t_ref, inclusive
        ds = [dd for _, dd in got]
        exp, window = [], []
        for t, dd in enumerate(ds):
            window.append(dd)
            s = np.float32(0.0)
            for w in window:
                s = np.float32(s + np.float32(w))
            if s > np.float32(thr):
                exp.append(1)
                window = [dd]
            else:
                exp.append(0)
        assert [m for m, _ in got] == exp


# ---------------------------------------------------------------------------
# Gate-mask consumer: gather / scatter around the model forward
# ---------------------------------------------------------------------------
def test_gather_scatter_round_trip():
    rng = np.random.default_rng(21)
    x = rng.standard_normal((6, 10)).astype(np.float32)
    mask = np.array([0, 1, 1, 0, 0, 1], np.uint8)
    ids, count, dense = O.gather_recompute(x, mask)
    assert count == 3 and list(ids) == [1, 2, 5, -1, -1, -1]
    np.testing.assert_array_equal(dense[:3], x[[1, 2, 5]])
    assert np.all(dense[3:] == 0)
    v_cache = rng.standard_normal((6, 10)).astype(np.float32)
    fresh = rng.standard_normal((6, 10)).astype(np.float32)
    out = O.scatter_velocity(v_cache, fresh, ids, count)
    np.testing.assert_array_equal(out[[1, 2, 5]], fresh[:3])
    np.testing.assert_array_equal(out[[0, 3, 4]], v_cache[[0, 3, 4]])
    ids0, c0, d0 = O.gather_recompute(x, np.zeros(6, np.uint8))
    assert c0 == 0 and np.all(ids0 == -1) and np.all(d0 == 0)


# ---- cache buffer management -------------------------------------------------

def _stream_inputs(H, C, d, n_chunks, Lq, seed, same_query=False):
    rng = np.random.default_rng(seed)
    ks = [rng.standard_normal((H, C, d)) for _ in range(n_chunks)]
    vs = [rng.standard_normal((H, C, d)) for _ in range(n_chunks)]
    if same_query:
        q0 = rng.standard_normal((H, 1, d))
        qs = [np.repeat(q0, Lq, axis=1) for _ in range(n_chunks)]
    else:
        qs = [rng.standard_normal((H, Lq, d)) for _ in range(n_chunks)]
    return ks, vs, qs


def test_cache_fills_then_holds_the_budget():
    """The clean length grows by one chunk while it fits, then stays at
    B_budget; before the first compression the buffer is the chunks in order."""
    H, C, d, B = 2, 4, 8, 12
    ks, vs, qs = _stream_inputs(H, C, d, 7, 3, seed=0)
    _, _, n, lengths = O.cache_stream(ks, vs, qs, B, 0.5, 3)
    assert lengths == [4, 8, 12, 12, 12, 12, 12] and n == 12
    kb, vb, n, _ = O.cache_stream(ks[:3], vs[:3], qs[:3], B, 0.5, 3)
    np.testing.assert_array_equal(kb[:, :12], np.concatenate(ks[:3], axis=1))
    np.testing.assert_array_equal(vb[:, :12], np.concatenate(vs[:3], axis=1))


def test_cache_ragged_chunks_fill_to_the_budget():
    """A chunk size that does not divide the budget: the clean length grows by
    C while n + C fits, the first overflow compresses n + C < B + C candidates
    down to B, and from then on every chunk brings B + C candidates."""
    H, C, d, B = 2, 5, 8, 12
    ks, vs, qs = _stream_inputs(H, C, d, 6, 3, seed=2)
    _, _, n, lengths = O.cache_stream(ks, vs, qs, B, 0.5, 3)
    assert lengths == [5, 10, 12, 12, 12, 12] and n == 12
    kb = np.zeros((H, B + C, d))
    vb = np.zeros((H, B + C, d))
    kb[:, :15] = np.concatenate(ks[:3], axis=1)
    vb[:, :15] = np.concatenate(vs[:3], axis=1)
    kn, vn, n, idx = O.cache_commit(kb, vb, 10, C, B, qs[2], 0.5, 3)
    assert n == 12 and idx.shape == (H, 12) and idx.max() < 15
    for h in range(H):
        np.testing.assert_array_equal(kn[h, :12], kb[h, idx[h]])


@pytest.mark.parametrize("C,B", [(4, 8), (3, 8), (5, 7)])
def test_cache_importance_only_keeps_global_top_b_by_dot_product(C, B):
    """lambda = 1, no pooling and one query repeated: the softmax is monotone
    in q.k, so each compression keeps the B largest q.k among its candidates,
    and over the stream the clean set is the B largest q.k of all tokens seen,
    in the order they arrived (brute force over the concatenated tokens).
    Holds whether or not C divides B."""
    H, d, n_chunks = 3, 8, 6
    ks, vs, qs = _stream_inputs(H, C, d, n_chunks, 5, seed=1, same_query=True)
    kb, vb, n, _ = O.cache_stream(ks, vs, qs, B, 1.0, 1)
    allk = np.concatenate(ks, axis=1)
    allv = np.concatenate(vs, axis=1)
    for h in range(H):
        dots = allk[h] @ qs[0][h, 0]
        keep = np.sort(np.argsort(-dots)[:B])
        np.testing.assert_array_equal(kb[h, :B], allk[h, keep])
        np.testing.assert_array_equal(vb[h, :B], allv[h, keep])


def test_cache_redundancy_only_drops_the_repeated_key():
    """lambda = 0: the score is minus the redundancy.  Candidates
    [e1, e1, e2, e1, e3, e4]: each copy of e1 has cosine row sum 2, the others
    0, so the three kept are e2, e3, e4 (candidate rows 2, 4, 5)."""
    e = np.eye(4)
    k1 = np.stack([e[0], e[0], e[1]])[None]
    k2 = np.stack([e[0], e[2], e[3]])[None]
    v1, v2 = k1 * 10, k2 * 10
    q = np.ones((1, 2, 4))
    kb = np.zeros((1, 6, 4))
    vb = np.zeros((1, 6, 4))
    kb[:, :3], vb[:, :3] = k1, v1
    kb, vb, n, idx = O.cache_commit(kb, vb, 0, 3, 3, q, 0.0, 1)
    assert n == 3 and idx is None
    kb[:, 3:], vb[:, 3:] = k2, v2
    kn, vn, n, idx = O.cache_commit(kb, vb, 3, 3, 3, q, 0.0, 1)
    assert n == 3
    np.testing.assert_array_equal(idx, [[2, 4, 5]])
    np.testing.assert_array_equal(kn[0, :3], np.stack([e[1], e[2], e[3]]))
    np.testing.assert_array_equal(vn[0, :3], 10 * np.stack([e[1], e[2], e[3]]))
    assert not kn[:, 3:].any()
