"""Helpers shared by the GPU parity tests: run the library through its
C-ABI binding on torch CUDA tensors and return numpy results, plus the
comparison rules (tolerances and margin waivers) the tests apply."""

import numpy as np
import torch

import cache_gating_kv_b200 as fc

DEV = "cuda"

# Score tolerances: float32 inputs agree to 1e-5 relative to the head's largest
# |score|; bf16 inputs (fp32 accumulation) to 2e-3 of the head's score range.
TOL_F32 = 1e-5
TOL_BF16 = 2e-3


def gate_gpu(x, v, dt, step, m, eps, f, ws=None):
    """One gate step on the GPU; returns numpy (x_next, f_next, l1, mask)."""
    xd = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(DEV)
    vd = torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(DEV)
    n_c = xd.shape[0]
    dtd = torch.from_numpy(np.asarray(dt, np.float32)).to(DEV)
    sd = torch.from_numpy(np.asarray(step, np.int32)).to(DEV)
    fd = torch.from_numpy(np.asarray(f, np.float32).copy()).to(DEV)
    l1 = torch.full((n_c,), -1.0, device=DEV)
    mask = torch.full((n_c,), 7, dtype=torch.uint8, device=DEV)
    if ws is None:
        ws = fc.workspace(fc.fc_gate_workspace_size(n_c, xd.shape[1]))
    fc.fc_chunk_l1_gate(xd, vd, dtd, sd, m, eps, fd, l1, mask, ws)
    torch.cuda.synchronize()
    return xd.cpu().numpy(), fd.cpu().numpy(), l1.cpu().numpy(), mask.cpu().numpy()


def importance_gpu(q, k, scale=0.0):
    H, Lq, d = q.shape
    Lk = k.shape[1]
    code = fc.FC_BF16 if q.dtype == torch.bfloat16 else fc.FC_F32
    imp = torch.full((H, Lk), -1.0, device=DEV)
    ws = fc.workspace(fc.fc_importance_workspace_size(code, H, Lq, Lk, d))
    fc.fc_kv_importance(q.to(DEV), k.to(DEV), imp, ws, scale=scale)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0, "a bounded device wait gave up"
    return imp.cpu().numpy()


def redundancy_gpu(k):
    H, Lk, d = k.shape
    code = fc.FC_BF16 if k.dtype == torch.bfloat16 else fc.FC_F32
    red = torch.full((H, Lk), -1.0, device=DEV)
    ws = fc.workspace(fc.fc_redundancy_workspace_size(code, H, Lk, d))
    fc.fc_kv_redundancy(k.to(DEV), red, ws)
    torch.cuda.synchronize()
    return red.cpu().numpy()


def score_topb_gpu(imp, red, pool, lam, B, want_score=True):
    H, Lk = imp.shape
    imp_d = torch.from_numpy(np.ascontiguousarray(imp, np.float32)).to(DEV)
    red_d = torch.from_numpy(np.ascontiguousarray(red, np.float32)).to(DEV)
    idx = torch.full((H, B), -7, dtype=torch.int32, device=DEV)
    score = torch.full((H, Lk), np.nan, device=DEV) if want_score else None
    ws = fc.workspace(fc.fc_score_topb_workspace_size(H, Lk, B))
    fc.fc_kv_score_topb(imp_d, red_d, pool, lam, B, idx, ws, score=score)
    torch.cuda.synchronize()
    return (score.cpu().numpy() if want_score else None), idx.cpu().numpy()


def compact_gpu(k, v, idx):
    H, Lk, d = k.shape
    B = idx.shape[1]
    kd, vd = k.to(DEV), v.to(DEV)
    ko = torch.full((H, B, d), 3.0, dtype=k.dtype, device=DEV)
    vo = torch.full((H, B, d), 3.0, dtype=k.dtype, device=DEV)
    fc.fc_kv_compact(kd, vd, torch.from_numpy(np.ascontiguousarray(idx, np.int32)).to(DEV), ko, vo)
    torch.cuda.synchronize()
    return ko.cpu(), vo.cpu()


def f64(t):
    return t.float().numpy().astype(np.float64)


def assert_selection_matches(idx_gpu, score_ref, B, tol):
    """Index sets must be identical except for tokens whose reference score is
    within ``tol`` of the reference B-th score (the margin waiver)."""
    H, Lk = score_ref.shape
    for h in range(H):
        g = idx_gpu[h]
        assert np.all(np.diff(g[g >= 0]) > 0), "indices must be strictly ascending"
        if B >= Lk:
            continue
        thr = np.sort(score_ref[h])[::-1][B - 1]
        gs = set(g.tolist())
        ref_keep = np.flatnonzero(score_ref[h] > thr + tol)
        ref_drop = np.flatnonzero(score_ref[h] < thr - tol)
        assert gs.issuperset(ref_keep.tolist()), f"head {h}: a clear keeper was dropped"
        assert not gs.intersection(ref_drop.tolist()), f"head {h}: a clear loser was kept"
        assert len(gs) == B


def history_gate_gpu(h_old, h_new, step, m, delta, f, ws=None):
    """One history-gate step on the GPU; returns numpy (h_next, f_next, d, refresh)."""
    ho = torch.from_numpy(np.ascontiguousarray(h_old, np.float32)).to(DEV)
    hn = torch.from_numpy(np.ascontiguousarray(h_new, np.float32)).to(DEV)
    n = ho.shape[0]
    sd = torch.from_numpy(np.asarray(step, np.int32)).to(DEV)
    fd = torch.from_numpy(np.asarray(f, np.float32).copy()).to(DEV)
    d = torch.full((n,), -1.0, device=DEV)
    r = torch.full((n,), 7, dtype=torch.uint8, device=DEV)
    if ws is None:
        ws = fc.workspace(fc.fc_gate_workspace_size(n, ho.shape[1]))
    fc.fc_history_l1_gate(ho, hn, sd, m, delta, fd, d, r, ws)
    torch.cuda.synchronize()
    return ho.cpu().numpy(), fd.cpu().numpy(), d.cpu().numpy(), r.cpu().numpy()
