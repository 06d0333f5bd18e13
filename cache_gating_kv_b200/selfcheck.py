"""Installation check: ``python -m cache_gating_kv_b200.selfcheck``.

Runs every call of the library once on the current GPU with small random
inputs and checks properties that hold exactly or nearly so without a
reference implementation: the gate's Euler update equals torch's
``x + v*dt`` (one rounding each), L1_rel is the ratio of the two L1 norms,
rows of the importance and the redundancy sum to one, the selection is
ascending, in range and a top-B of the returned scores, the compaction equals
``index_select`` bitwise, the mask consumer round-trips, a cache commit keeps
rows of its candidates, and no bounded device wait gave up.  Exits non-zero
and names the first failed check.
"""

import sys

import torch

import cache_gating_kv_b200 as fc


def _check(cond, what):
    if not cond:
        raise AssertionError(what)
    print(f"  ok  {what}")


def run(device=0):
    if not torch.cuda.is_available():
        raise SystemExit("selfcheck needs a CUDA device")
    dev = torch.device("cuda", device)
    torch.cuda.set_device(dev)
    g = torch.Generator(device="cpu").manual_seed(0)
    print(f"libflowcache {fc.fc_version()} on {torch.cuda.get_device_name(dev)}")

    # gate
    n_c, N = 5, 10007
    x = torch.randn(n_c, N, generator=g).to(dev)
    v = torch.randn(n_c, N, generator=g).to(dev)
    dt = torch.tensor([-0.02, -0.01, -0.05, 0.0, -0.03], device=dev)
    step = torch.tensor([0, 3, 4, -1, 7], dtype=torch.int32, device=dev)
    f = torch.zeros(n_c, device=dev)
    l1 = torch.empty(n_c, device=dev)
    mask = torch.empty(n_c, dtype=torch.uint8, device=dev)
    ws = fc.workspace(fc.fc_gate_workspace_size(n_c, N), dev)
    x0 = x.clone()
    fc.fc_chunk_l1_gate(x, v, dt, step, 2, 0.05, f, l1, mask, ws)
    torch.cuda.synchronize()
    upd = v * dt[:, None]
    want = x0 + upd
    act = step >= 0
    _check(torch.equal(x[act], want[act]) and torch.equal(x[~act], x0[~act]),
           "gate: X <- X + v*dt bitwise, inactive chunks untouched")
    ratio = upd.double().abs().sum(1) / x0.double().abs().sum(1)
    _check(torch.allclose(l1[act].double(), ratio[act], rtol=1e-6),
           "gate: L1_rel = ||v*dt||_1 / ||X_t||_1")
    _check(bool(mask[0]) and mask[3] == 0, "gate: forced step recomputes, inactive chunk reuses")
    _check(fc.fc_check_workspace(fc.FC_WS_GATE, ws, n_c), "gate: no bounded wait gave up")

    # mask consumer
    dense = torch.empty_like(x)
    ids = torch.empty(n_c, dtype=torch.int32, device=dev)
    cnt = torch.empty(1, dtype=torch.int32, device=dev)
    fc.fc_gather_recompute(x, mask, dense, ids, cnt)
    torch.cuda.synchronize()
    sel = torch.nonzero(mask).flatten()
    c = int(cnt.item())
    _check(c == sel.numel() and torch.equal(ids[:c].long(), sel) and
           torch.equal(dense[:c], x[sel]), "gather: the recompute chunks in order")
    vc = v.clone()
    fc.fc_scatter_velocity(dense, ids, cnt, vc)
    torch.cuda.synchronize()
    want_v = v.clone()
    want_v[sel] = x[sel]
    _check(torch.equal(vc, want_v), "scatter: fresh rows in, reused rows kept")

    # compression chain
    H, Lq, Lk, d, B = 3, 300, 2000, 128, 700
    q = torch.randn(H, Lq, d, generator=g).to(torch.bfloat16).to(dev)
    k = torch.randn(H, Lk, d, generator=g).to(torch.bfloat16).to(dev)
    vv = torch.randn(H, Lk, d, generator=g).to(torch.bfloat16).to(dev)
    imp = torch.empty(H, Lk, device=dev)
    red = torch.empty(H, Lk, device=dev)
    sc = torch.empty(H, Lk, device=dev)
    idx = torch.empty(H, B, dtype=torch.int32, device=dev)
    ko = torch.empty(H, B, d, dtype=torch.bfloat16, device=dev)
    vo = torch.empty_like(ko)
    wi = fc.workspace(fc.fc_importance_workspace_size(fc.FC_BF16, H, Lq, Lk, d), dev)
    fc.fc_kv_importance(q, k, imp, wi)
    fc.fc_kv_redundancy(k, red, fc.workspace(fc.fc_redundancy_workspace_size(fc.FC_BF16, H, Lk,
                                                                            d), dev))
    fc.fc_kv_score_topb(imp, red, 7, 0.5, B, idx,
                        fc.workspace(fc.fc_score_topb_workspace_size(H, Lk, B), dev), score=sc)
    fc.fc_kv_compact(k, vv, idx, ko, vo)
    torch.cuda.synchronize()
    _check(torch.allclose(imp.double().sum(1), torch.ones(H, dtype=torch.float64, device=dev),
                          rtol=1e-4), "importance: rows sum to one")
    _check(fc.fc_check_workspace(fc.FC_WS_IMPORTANCE, wi), "importance: no bounded wait gave up")
    _check(torch.allclose(red.double().sum(1), torch.ones(H, dtype=torch.float64, device=dev),
                          rtol=1e-5), "redundancy: rows sum to one")
    il = idx.long()
    _check(bool(((il[:, 1:] - il[:, :-1]) > 0).all()) and int(il.min()) >= 0 and
           int(il.max()) < Lk, "top-B: ascending, in range")
    kept = torch.gather(sc, 1, il)
    drop = sc.clone()
    drop.scatter_(1, il, float("-inf"))
    _check(bool((kept.min(1).values >= drop.max(1).values).all()),
           "top-B: no dropped score above a kept one")
    _check(all(torch.equal(ko[h], k[h].index_select(0, il[h])) and
               torch.equal(vo[h], vv[h].index_select(0, il[h])) for h in range(H)),
           "compaction: the kept rows, bitwise")

    # cache commit
    C, Bb = 500, 1500
    kb = k[:, :Bb + C].contiguous()
    vb = vv[:, :Bb + C].contiguous()
    kn, vn = torch.empty_like(kb), torch.empty_like(vb)
    cidx = torch.empty(H, Bb, dtype=torch.int32, device=dev)
    cws = fc.workspace(fc.fc_kv_cache_workspace_size(fc.FC_BF16, H, Lq, Bb, C, d), dev)
    n, comp = fc.fc_kv_cache_commit(q, kb, vb, kn, vn, Bb, C, cws, 7, 0.5, idx=cidx)
    torch.cuda.synchronize()
    cl = cidx.long()
    _check(comp and n == Bb and all(torch.equal(kn[h, :Bb], kb[h].index_select(0, cl[h]))
                                    for h in range(H)),
           "cache commit: a full buffer compresses to B_budget candidate rows")
    _check(fc.fc_check_workspace(fc.FC_WS_CACHE, cws), "cache commit: no bounded wait gave up")
    print("selfcheck passed")


def main():
    try:
        run()
    except AssertionError as e:
        print(f"  FAILED  {e}")
        sys.exit(1)


if __name__ == "__main__":
    main()
