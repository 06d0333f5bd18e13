"""Full-size GPU checks: the long-history layer (H=40, L_q=8192, L_k=131072,
B=32768, 25% exact duplicate keys) and the full-step sweep layers (H=40,
L_q=4096, L_k up to 131072, B=L_k/4), launched exactly as bench.py launches
the calls (every head of the layer at once).

- One head of every layer goes through the oracle in full (the whole softmax
  of every query row, the whole L_k x L_k cosine matrix): its importance and
  redundancy are compared element by element, its score vector within 2e-3 of
  the head's score range, and its selected index set with the margin waiver
  (tokens whose oracle score is within that tolerance of the B-th score).
- Every head is checked against properties that hold at any size: rows of
  Imp and Red sum to one; exact duplicate keys get bitwise-equal importance and
  redundancy; idx is strictly ascending, in range, and a top-B selection of the
  returned scores with ties kept lowest-index-first; the compacted rows are the
  selected rows, bitwise."""

import numpy as np
import pytest
import torch

from cache_gating_kv_b200 import workloads as W
from oracle import flowcache_oracle as O
from tests.gpu_util import (TOL_BF16, assert_selection_matches, compact_gpu, f64, importance_gpu,
                            redundancy_gpu, score_topb_gpu)

pytestmark = pytest.mark.gpu


def _check_topb_properties(sc, idx, B):
    H, Lk = sc.shape
    for h in range(H):
        sel = idx[h]
        assert np.all(np.diff(sel) > 0) and sel[0] >= 0 and sel[-1] < Lk
        mask = np.zeros(Lk, bool)
        mask[sel] = True
        kept, dropped = sc[h][mask], sc[h][~mask]
        if dropped.size:
            lo, hi = kept.min(), dropped.max()
            assert lo >= hi, f"head {h}: a kept score {lo} is below a dropped one {hi}"
            if lo == hi:  # ties at the threshold: the kept ones have the lowest indices
                tie = np.flatnonzero(sc[h] == lo)
                kept_tie = np.flatnonzero(mask & (sc[h] == lo))
                np.testing.assert_array_equal(kept_tie, tie[:kept_tie.size])


def _check_head_against_oracle(q, k, imp, red, sc, idx, h, cfg, lam):
    """Head h through the oracle in full: Imp and Red element by element (bf16
    inputs: 1e-4 relative plus 1e-4 of the head's largest value for Imp; Red
    is formed from the same bf16 values in float32, 1e-5 relative), the score
    within 2e-3 of the head's score range, the selection up to the margin
    waiver."""
    qh, kh = f64(q[h:h + 1]), f64(k[h:h + 1])
    imp_r = O.importance(qh, kh)[0]
    red_r = O.redundancy(kh)[0]
    got_i = imp[h].astype(np.float64)
    assert np.all(np.abs(got_i - imp_r) <= 1e-4 * imp_r + 1e-4 * imp_r.max()), \
        float(np.max(np.abs(got_i - imp_r) / imp_r))
    np.testing.assert_allclose(red[h].astype(np.float64), red_r, rtol=1e-5, atol=0)
    sc_r = O.score(imp_r[None], red_r[None], lam, cfg.pool)
    span = float(sc_r.max() - sc_r.min())
    assert np.max(np.abs(sc[h].astype(np.float64) - sc_r[0])) <= TOL_BF16 * span
    assert_selection_matches(idx[h:h + 1], sc_r.astype(np.float64), cfg.B, TOL_BF16 * span)


def _run_layer(cfg, layer, heads_for_oracle, seed=0):
    q, k, v = W.kv_inputs(cfg, seed=seed, layer=layer)
    imp = importance_gpu(q, k)
    red = redundancy_gpu(k)
    lam = cfg.lam[len(cfg.lam) // 2]
    sc, idx = score_topb_gpu(imp, red, cfg.pool, lam, cfg.B)
    np.testing.assert_allclose(imp.sum(axis=1), 1.0, rtol=3e-4)
    np.testing.assert_allclose(red.sum(axis=1), 1.0, rtol=1e-5)
    _check_topb_properties(sc, idx, cfg.B)
    ko, vo = compact_gpu(k, v, idx)
    for h in (0, cfg.H // 2, cfg.H - 1):
        sel = torch.from_numpy(idx[h].astype(np.int64))
        assert torch.equal(ko[h], k[h].index_select(0, sel))
        assert torch.equal(vo[h], v[h].index_select(0, sel))
    for h in heads_for_oracle:
        _check_head_against_oracle(q, k, imp, red, sc, idx, h, cfg, lam)
    return q, k, imp, red, sc, idx


def test_long_history_layer_full_size():
    cfg = W.KV_CONFIGS["long_history"]
    q, k, imp, red, sc, idx = _run_layer(cfg, 0, heads_for_oracle=[0])
    # exact duplicate K rows: bitwise-equal importance and redundancy
    for h in (0, 17, 39):
        kh = k[h].view(torch.int16).numpy()
        _, first, inverse = np.unique(kh, axis=0, return_index=True, return_inverse=True)
        twin = first[inverse.ravel()]
        dup = np.flatnonzero(twin != np.arange(cfg.Lk))
        assert dup.size > cfg.Lk // 5  # the workload makes 25 % duplicates
        np.testing.assert_array_equal(imp[h, dup].view(np.uint32), imp[h, twin[dup]].view(np.uint32))
        np.testing.assert_array_equal(red[h, dup].view(np.uint32), red[h, twin[dup]].view(np.uint32))


@pytest.mark.parametrize("Lk", [4096, 16384, 65536, 131072])
def test_full_step_sweep_layer(Lk):
    cfg = W.KV_CONFIGS[f"sweep_lk{Lk}"]
    _run_layer(cfg, layer=Lk % 40, heads_for_oracle=[0])
