"""GPU parity of fc_kv_cache_commit (cache buffer management around
compression) with the oracle's cache_commit / cache_stream.

- float32 stream: every commit against the oracle (selection exact, the
  clean rows bitwise), on a seed whose selection margins the oracle shows to
  be clear of the float32 tolerance;
- bf16 first compression: the selection against the oracle under the margin
  waiver, the kept rows bitwise, the next chunk's rows untouched;
- bf16 stream: every commit equals the separate calls (importance,
  redundancy, score/top-B, compaction) on the same buffer, bitwise;
- bf16 stream with lambda = 1, no pooling and one query repeated: the final
  clean set is the global top-B_budget by q.k (brute force in float64);
- streams whose chunk size does not divide the budget (both dtypes): the
  clean counts follow the oracle's, every compression selects under the
  margin waiver from exactly the n_clean + C candidates (the buffer rows past
  them are NaN) and keeps those rows bitwise."""

import numpy as np
import pytest
import torch

import cache_gating_kv_b200 as fc
from cache_gating_kv_b200 import workloads as W
from oracle import flowcache_oracle as O
from tests.gpu_util import DEV, TOL_BF16, TOL_F32, assert_selection_matches, f64

pytestmark = pytest.mark.gpu


class GpuCache:
    """Two preallocated buffers [H, B_budget + C, d]; commit swaps them when
    the library reports a compression."""

    def __init__(self, H, C, B, d, Lq, dtype, sentinel=0.0):
        self.H, self.C, self.B, self.d = H, C, B, d
        cap = B + C
        self.bufs = [(torch.full((H, cap, d), sentinel, dtype=dtype, device=DEV),
                      torch.full((H, cap, d), sentinel, dtype=dtype, device=DEV)) for _ in range(2)]
        self.cur = 0
        self.n = 0
        code = fc.FC_BF16 if dtype == torch.bfloat16 else fc.FC_F32
        self.ws = fc.workspace(fc.fc_kv_cache_workspace_size(code, H, Lq, B, C, d))
        self.idx = torch.full((H, B), -7, dtype=torch.int32, device=DEV)

    def write_chunk(self, k, v):
        kb, vb = self.bufs[self.cur]
        kb[:, self.n:self.n + self.C] = k.to(DEV)
        vb[:, self.n:self.n + self.C] = v.to(DEV)

    def commit(self, q, lam, pool):
        kb, vb = self.bufs[self.cur]
        kn, vn = self.bufs[1 - self.cur]
        self.n, comp = fc.fc_kv_cache_commit(q.to(DEV), kb, vb, kn, vn, self.n, self.C, self.ws,
                                             pool, lam, idx=self.idx)
        if comp:
            self.cur = 1 - self.cur
        assert int(self.ws[:4].view(torch.int32).item()) == 0, "a bounded device wait gave up"
        return comp

    def clean(self):
        kb, vb = self.bufs[self.cur]
        return kb[:, :self.n].cpu(), vb[:, :self.n].cpu()


def _oracle_commit_with_scores(kb, vb, n, C, B, q, lam, pool):
    """The oracle's commit plus its score of the candidates (for margins)."""
    out = O.cache_commit(kb, vb, n, C, B, q, lam, pool)
    sc = None
    if out[3] is not None:
        L = n + C
        sc = O.score(O.importance(q, kb[:, :L]), O.redundancy(kb[:, :L]), lam, pool)
    return out, sc


def _margin(sc, B):
    """Smallest gap, over heads, between the B-th and (B+1)-th score, relative
    to the head's largest |score|."""
    gaps = []
    for h in range(sc.shape[0]):
        s = np.sort(sc[h].astype(np.float64))[::-1]
        gaps.append((s[B - 1] - s[B]) / np.abs(s).max())
    return min(gaps)


def test_fp32_stream_matches_oracle():
    cfg = W.CACHE_CONFIGS["tiny_fp32_stream"]
    ks, vs, qs = W.cache_inputs(cfg, seed=2)
    H, C, B, d = cfg.H, cfg.C, cfg.B_budget, cfg.d
    g = GpuCache(H, C, B, d, cfg.Lq, torch.float32, sentinel=float("nan"))
    kb = np.zeros((H, B + C, d))
    vb = np.zeros((H, B + C, d))
    n = 0
    n_compressions = 0
    for i in range(cfg.n_chunks):
        kb = kb.copy()
        vb = vb.copy()
        kb[:, n:n + C], vb[:, n:n + C] = f64(ks[i]), f64(vs[i])
        (kb, vb, n, idx_ref), sc = _oracle_commit_with_scores(kb, vb, n, C, B, f64(qs[i]),
                                                              cfg.lam, cfg.pool)
        g.write_chunk(ks[i], vs[i])
        comp = g.commit(qs[i], cfg.lam, cfg.pool)
        assert g.n == n and comp == (idx_ref is not None)
        if comp:
            n_compressions += 1
            assert _margin(sc, B) > 4 * TOL_F32, "pick a seed with clear margins"
            np.testing.assert_array_equal(g.idx.cpu().numpy(), idx_ref)
        gk, gv = g.clean()
        np.testing.assert_array_equal(gk.numpy().astype(np.float64), kb[:, :n])
        np.testing.assert_array_equal(gv.numpy().astype(np.float64), vb[:, :n])
    assert n_compressions == cfg.n_chunks - B // C


def test_bf16_first_compression_matches_oracle():
    cfg = W.CACHE_CONFIGS["bf16_stream"]
    ks, vs, qs = W.cache_inputs(cfg, seed=1)
    H, C, B, d = cfg.H, cfg.C, cfg.B_budget, cfg.d
    g = GpuCache(H, C, B, d, cfg.Lq, torch.bfloat16, sentinel=7.0)
    n_fill = B // C
    for i in range(n_fill):
        g.write_chunk(ks[i], vs[i])
        assert not g.commit(qs[i], cfg.lam, cfg.pool)
        assert fc.fc_last_launches() == 0
    g.write_chunk(ks[n_fill], vs[n_fill])
    kb_before = g.bufs[g.cur][0].cpu()
    vb_before = g.bufs[g.cur][1].cpu()
    q = qs[n_fill]
    assert g.commit(q, cfg.lam, cfg.pool) and g.n == B
    idx = g.idx.cpu().numpy()
    kn, vn = g.bufs[g.cur]
    # the next chunk's rows of the new buffer are not written
    assert torch.all(kn[:, B:] == 7.0) and torch.all(vn[:, B:] == 7.0)
    # the kept rows are the candidates at idx, bitwise, in order
    for h in range(H):
        sel = torch.from_numpy(idx[h].astype(np.int64))
        assert torch.equal(kn[h, :B].cpu(), kb_before[h].index_select(0, sel))
        assert torch.equal(vn[h, :B].cpu(), vb_before[h].index_select(0, sel))
    # the selection against the oracle's, under the bf16 margin waiver
    kc = f64(kb_before)
    sc_ref = O.score(O.importance(f64(q), kc), O.redundancy(kc), cfg.lam, cfg.pool)
    rng = sc_ref.max(axis=1) - sc_ref.min(axis=1)
    for h in range(H):
        assert_selection_matches(idx[h:h + 1], sc_ref[h:h + 1], B, TOL_BF16 * rng[h])


def test_bf16_stream_equals_separate_calls():
    cfg = W.CACHE_CONFIGS["bf16_stream"]
    ks, vs, qs = W.cache_inputs(cfg, seed=2)
    H, C, B, d = cfg.H, cfg.C, cfg.B_budget, cfg.d
    cap = B + C
    g = GpuCache(H, C, B, d, cfg.Lq, torch.bfloat16)
    ws_i = fc.workspace(fc.fc_importance_workspace_size(fc.FC_BF16, H, cfg.Lq, cap, d))
    ws_r = fc.workspace(fc.fc_redundancy_workspace_size(fc.FC_BF16, H, cap, d))
    ws_s = fc.workspace(fc.fc_score_topb_workspace_size(H, cap, B))
    compressions = 0
    for i in range(cfg.n_chunks):
        g.write_chunk(ks[i], vs[i])
        kb, vb = g.bufs[g.cur]
        kb0, vb0 = kb.clone(), vb.clone()
        q = qs[i].to(DEV)
        n_before = g.n
        comp = g.commit(q, cfg.lam, cfg.pool)
        if not comp:
            assert g.n == n_before + C
            continue
        compressions += 1
        imp = torch.empty(H, cap, device=DEV)
        red = torch.empty(H, cap, device=DEV)
        idx = torch.empty(H, B, dtype=torch.int32, device=DEV)
        fc.fc_kv_importance(q, kb0, imp, ws_i)
        fc.fc_kv_redundancy(kb0, red, ws_r)
        fc.fc_kv_score_topb(imp, red, cfg.pool, cfg.lam, B, idx, ws_s)
        ko = torch.empty(H, B, d, dtype=torch.bfloat16, device=DEV)
        vo = torch.empty_like(ko)
        fc.fc_kv_compact(kb0, vb0, idx, ko, vo)
        torch.cuda.synchronize()
        assert torch.equal(g.idx, idx)
        kn, vn = g.bufs[g.cur]
        assert torch.equal(kn[:, :B], ko) and torch.equal(vn[:, :B], vo)
    assert compressions == cfg.n_chunks - B // C


def test_bf16_importance_only_keeps_global_top_b():
    """lambda = 1, window 1, one query repeated: every compression keeps the
    B largest q.k among its candidates, so the final clean set is the B
    largest q.k of the whole stream (brute force in float64).  Tokens within
    1e-3 of the global B-th q.k may go either way (the rounding of the GPU's
    float32 softmax is about 1e-4 in q.k units); every other token must be
    decided as the brute force decides it."""
    cfg = W.CACHE_CONFIGS["bf16_stream"]
    ks, vs, qs = W.cache_inputs(cfg, seed=3)
    H, C, B, d = cfg.H, cfg.C, cfg.B_budget, cfg.d
    q1 = qs[0][:, :1].expand(H, cfg.Lq, d).contiguous()  # one query repeated
    allk = torch.cat(ks, dim=1)
    allv = torch.cat(vs, dim=1)
    dots = np.einsum("hld,hd->hl", f64(allk), f64(q1[:, 0]))
    g = GpuCache(H, C, B, d, cfg.Lq, torch.bfloat16)
    pos = np.zeros((H, 0), np.int64)  # stream position of every clean row
    for i in range(cfg.n_chunks):
        g.write_chunk(ks[i], vs[i])
        cand = np.concatenate([pos, np.tile(np.arange(i * C, (i + 1) * C), (H, 1))], axis=1)
        if g.commit(q1, 1.0, 1):
            pos = np.take_along_axis(cand, g.idx.cpu().numpy().astype(np.int64), axis=1)
        else:
            pos = cand
    assert pos.shape == (H, B)
    assert_selection_matches(pos, dots, B, 1e-3)
    gk, gv = g.clean()
    for h in range(H):
        sel = torch.from_numpy(pos[h])
        assert torch.equal(gk[h], allk[h].index_select(0, sel))
        assert torch.equal(gv[h], allv[h].index_select(0, sel))


@pytest.mark.parametrize("name", ["tiny_fp32_ragged", "bf16_ragged"])
def test_ragged_chunk_stream(name):
    cfg = W.CACHE_CONFIGS[name]
    ks, vs, qs = W.cache_inputs(cfg, seed=4)
    H, C, B, d = cfg.H, cfg.C, cfg.B_budget, cfg.d
    bf16 = cfg.dtype == "bf16"
    dtype = torch.bfloat16 if bf16 else torch.float32
    tol = TOL_BF16 if bf16 else TOL_F32
    g = GpuCache(H, C, B, d, cfg.Lq, dtype, sentinel=float("nan"))
    n_ref = 0
    sizes = []
    for i in range(cfg.n_chunks):
        g.write_chunk(ks[i], vs[i])
        L = g.n + C
        kb0, vb0 = (t[:, :L].cpu() for t in g.bufs[g.cur])
        comp = g.commit(qs[i], cfg.lam, cfg.pool)
        # the oracle's clean count for the same stream
        n_ref = n_ref + C if n_ref + C <= B else B
        assert g.n == n_ref and comp == (L > B)
        if not comp:
            continue
        sizes.append(L)
        idx = g.idx.cpu().numpy()
        assert idx.min() >= 0 and idx.max() < L
        kc = f64(kb0)
        sc = O.score(O.importance(f64(qs[i]), kc), O.redundancy(kc), cfg.lam, cfg.pool)
        kn, vn = g.bufs[g.cur]
        for h in range(H):
            span = (sc[h].max() - sc[h].min()) if bf16 else np.abs(sc[h]).max()
            assert_selection_matches(idx[h:h + 1], sc[h:h + 1], B, tol * max(float(span), 1e-30))
            sel = torch.from_numpy(idx[h].astype(np.int64))
            assert torch.equal(kn[h, :B].cpu(), kb0[h].index_select(0, sel))
            assert torch.equal(vn[h, :B].cpu(), vb0[h].index_select(0, sel))
    # the first compression saw fewer than B_budget + C candidates, the rest all of them
    assert sizes[0] < B + C and all(s == B + C for s in sizes[1:]) and len(sizes) >= 2
