"""Parity of the mask consumer (gather of the recompute chunks, scatter of the
fresh velocities) with the oracle's plain definitions: bitwise, since both
are copies.  Covers all-reuse and all-recompute masks, a single chunk, empty
and ragged chunk sizes, unaligned rows, and the gate's own mask on the device."""

import numpy as np
import pytest
import torch

import cache_gating_kv_b200 as fc
from cache_gating_kv_b200 import workloads as W
from oracle import flowcache_oracle as O
from tests.gpu_util import DEV

pytestmark = pytest.mark.gpu


def _gather(x, mask):
    n_c, N = x.shape
    xd = torch.from_numpy(x).to(DEV)
    md = torch.from_numpy(mask).to(DEV)
    dense = torch.full((n_c, N), float("nan"), device=DEV)
    ids = torch.full((n_c,), 99, dtype=torch.int32, device=DEV)
    count = torch.full((1,), -5, dtype=torch.int32, device=DEV)
    fc.fc_gather_recompute(xd, md, dense, ids, count)
    torch.cuda.synchronize()
    return dense, ids, count


def _check(x, mask, seed):
    n_c, N = x.shape
    dense, ids, count = _gather(x, mask)
    ids_ref, cnt_ref, dense_ref = O.gather_recompute(x, mask)
    assert int(count.item()) == cnt_ref
    np.testing.assert_array_equal(ids.cpu().numpy(), ids_ref)
    got = dense.cpu().numpy()[:cnt_ref]
    np.testing.assert_array_equal(got.view(np.uint32), dense_ref[:cnt_ref].view(np.uint32))
    # rows past count are not written
    assert np.all(np.isnan(dense.cpu().numpy()[cnt_ref:]))

    rng = np.random.default_rng(seed)
    v_cache = rng.standard_normal((n_c, N)).astype(np.float32)
    v_dense = rng.standard_normal((n_c, N)).astype(np.float32)
    vc = torch.from_numpy(v_cache).to(DEV)
    fc.fc_scatter_velocity(torch.from_numpy(v_dense).to(DEV), ids, count, vc)
    torch.cuda.synchronize()
    ref = O.scatter_velocity(v_cache, v_dense, ids_ref, cnt_ref)
    np.testing.assert_array_equal(vc.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("n_c,N", [(1, 1), (1, 4096), (4, 3), (5, 4097), (16, 65536 + 12),
                                   (40, 12288), (33, 1000), (200, 257)])
@pytest.mark.parametrize("kind", ["random", "none", "all", "last"])
def test_gather_scatter_match_oracle(n_c, N, kind):
    rng = np.random.default_rng(n_c * 7919 + N)
    x = rng.standard_normal((n_c, N)).astype(np.float32)
    if kind == "random":
        mask = (rng.random(n_c) < 0.4).astype(np.uint8) * rng.integers(1, 256, n_c).astype(np.uint8)
    elif kind == "none":
        mask = np.zeros(n_c, np.uint8)
    elif kind == "all":
        mask = np.ones(n_c, np.uint8)
    else:
        mask = np.zeros(n_c, np.uint8)
        mask[-1] = 1
    _check(x, mask, seed=N)


def test_empty_chunks():
    n_c = 6
    mask = np.array([1, 0, 1, 1, 0, 0], np.uint8)
    x = np.zeros((n_c, 0), np.float32)
    dense, ids, count = _gather(x, mask)
    assert int(count.item()) == 3
    np.testing.assert_array_equal(ids.cpu().numpy(), [0, 2, 3, -1, -1, -1])


def _chain_inputs():
    cfg = W.GATE_CONFIGS["full_step_sweep"]
    eps = cfg.eps[0]
    x = W.gate_initial(cfg, seed=0)
    v = W.gate_velocity(cfg, seed=0)
    step = W.gate_step_counters(cfg, 45)
    dt = W.gate_dt(cfg, step)
    f = np.where(np.arange(cfg.n_chunks) % 2 == 0, 2 * eps, 0.0).astype(np.float32)
    return cfg, eps, x, v, step, dt, f


def test_chain_inputs_have_clear_margins():
    """The chain test below compares masks exactly: every active chunk's
    f + L1 is far from eps, and the mask mixes recompute and reuse."""
    cfg, eps, x, v, step, dt, f = _chain_inputs()
    _, _, l1, mask = O.gate_step(x, v, dt, step, cfg.m, eps, f)
    act = step >= cfg.m
    assert np.all(np.abs(f[act] + l1[act] - eps) > 1e-3 * eps)
    assert 0 < mask.sum() < cfg.n_chunks


def test_consumes_the_gate_mask_on_device():
    """gate -> gather -> (forward stand-in) -> scatter, without leaving the
    device, against the oracle's gate and consumer."""
    cfg, eps, x, v, step, dt, f = _chain_inputs()
    n_c, N = x.shape
    xd, vd = torch.from_numpy(x).to(DEV), torch.from_numpy(v).to(DEV)
    fd = torch.from_numpy(f.copy()).to(DEV)
    dtd = torch.from_numpy(dt).to(DEV)
    sd = torch.from_numpy(step).to(DEV)
    l1 = torch.empty(n_c, device=DEV)
    mask = torch.empty(n_c, dtype=torch.uint8, device=DEV)
    ws = fc.workspace(fc.fc_gate_workspace_size(n_c, N))
    fc.fc_chunk_l1_gate(xd, vd, dtd, sd, cfg.m, eps, fd, l1, mask, ws)
    dense = torch.empty_like(xd)
    ids = torch.empty(n_c, dtype=torch.int32, device=DEV)
    count = torch.empty(1, dtype=torch.int32, device=DEV)
    fc.fc_gather_recompute(xd, mask, dense, ids, count)
    v_fresh = dense * 0.5  # stands in for the model forward on the dense batch
    fc.fc_scatter_velocity(v_fresh, ids, count, vd)
    torch.cuda.synchronize()

    x_ref, _, _, m_ref = O.gate_step(x, v, dt, step, cfg.m, eps, f)
    np.testing.assert_array_equal(mask.cpu().numpy(), m_ref)
    ids_ref, cnt, dense_ref = O.gather_recompute(x_ref, m_ref)
    assert int(count.item()) == cnt
    np.testing.assert_array_equal(ids.cpu().numpy(), ids_ref)
    v_ref = O.scatter_velocity(v, (dense_ref * np.float32(0.5)).astype(np.float32), ids_ref, cnt)
    np.testing.assert_array_equal(vd.cpu().numpy().view(np.uint32), v_ref.view(np.uint32))
