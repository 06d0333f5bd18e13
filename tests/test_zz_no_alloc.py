"""The allocation-free gate entry point, fc_chunk_l1_gate_noalloc.

Some callers cannot allocate device memory when they run the gate (a host
runtime that gives a plugin only its input and output buffers and forbids
cudaMalloc while work is enqueued, or code with nowhere to keep a workspace
alive between steps).  For them the library keeps the gate's scratch in a
fixed static device array.  This test drives that entry point through the
C-ABI and checks that two calls in a row give what the workspace entry point
gives on the same inputs, within the gate tests' tolerances (bitwise update,
L1 to 1e-6 relative, exact masks and accumulators).

It sits in its own file that pytest collects last, and must pass both in a
fresh process and after every other test (the static scratch then holds what
earlier calls left in it).
"""

import numpy as np
import pytest
import torch

import cache_gating_kv_b200 as fc
from cache_gating_kv_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _state(x, v, dt, step, f):
    t = lambda a, dtype=None: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)  # noqa: E731
    n_c = x.shape[0]
    return {"x": t(x), "v": t(v), "dt": t(dt), "step": t(step), "f": t(f),
            "l1": torch.full((n_c,), -1.0, device=DEV),
            "mask": torch.full((n_c,), 7, dtype=torch.uint8, device=DEV)}


def _snapshot(s):
    torch.cuda.synchronize()
    return {k: s[k].cpu().numpy().copy() for k in ("x", "f", "l1", "mask")}


def _two_calls(x, v, dt, step, m, eps, f):
    """Two consecutive steps through each entry point from the same state."""
    a = _state(x, v, dt, step, f)
    b = _state(x, v, dt, step, f)
    ws = fc.workspace(fc.fc_gate_workspace_size(x.shape[0], x.shape[1]))
    out_a, out_b = [], []
    for _ in range(2):
        fc.fc_chunk_l1_gate(a["x"], a["v"], a["dt"], a["step"], m, eps, a["f"], a["l1"],
                            a["mask"], ws)
        out_a.append(_snapshot(a))
        fc.fc_chunk_l1_gate_noalloc(b["x"], b["v"], b["dt"], b["step"], m, eps, b["f"], b["l1"],
                                    b["mask"])
        out_b.append(_snapshot(b))
    return out_a, out_b


def _assert_same(out_a, out_b):
    for ra, rb in zip(out_a, out_b):
        np.testing.assert_array_equal(rb["x"].view(np.uint32), ra["x"].view(np.uint32))
        np.testing.assert_allclose(rb["l1"], ra["l1"], rtol=1e-6, atol=0)
        np.testing.assert_array_equal(rb["mask"], ra["mask"])
        np.testing.assert_allclose(rb["f"], ra["f"], rtol=1e-6, atol=0)


def test_noalloc_gate_matches_workspace_gate_twice_on_workload():
    cfg = W.GATE_CONFIGS["bf16_layer"]
    x = W.gate_initial(cfg, seed=7)
    v = W.gate_velocity(cfg, seed=7)
    step = np.full(cfg.n_chunks, cfg.m + 3, np.int32)
    dt = W.gate_dt(cfg, step)
    f = np.float32([0.0, 0.002, 0.004, 0.009])
    _assert_same(*_two_calls(x, v, dt, step, cfg.m, cfg.eps[0], f))


def test_noalloc_gate_at_its_chunk_limit_with_ragged_chunks():
    rng = np.random.default_rng(11)
    n_c, N = 32, 1003  # the largest chunk count it serves; misaligned chunk starts
    x = rng.standard_normal((n_c, N)).astype(np.float32)
    v = rng.standard_normal((n_c, N)).astype(np.float32)
    dt = rng.uniform(-0.05, 0.05, n_c).astype(np.float32)
    step = np.where(np.arange(n_c) % 5 == 0, -1, np.arange(n_c)).astype(np.int32)
    f = (rng.random(n_c) * 0.05).astype(np.float32)
    _assert_same(*_two_calls(x, v, dt, step, 2, 0.06, f))


def test_noalloc_gate_rejects_too_many_chunks_before_launch():
    n_c = 33
    s = _state(np.zeros((n_c, 8), np.float32), np.zeros((n_c, 8), np.float32),
               np.zeros(n_c, np.float32), np.zeros(n_c, np.int32), np.zeros(n_c, np.float32))
    with pytest.raises(fc.FlowCacheError, match="1 to 32 chunks"):
        fc.fc_chunk_l1_gate_noalloc(s["x"], s["v"], s["dt"], s["step"], 1, 0.1, s["f"], s["l1"],
                                    s["mask"])
    torch.cuda.synchronize()
    assert int(s["mask"][0]) == 7  # nothing was launched
