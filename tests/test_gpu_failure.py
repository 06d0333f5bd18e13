"""Failure detection on the GPU without a fault: the error word a bounded
device-side wait would set is read back by fc_check_workspace.  The word is
set here by the host (a planted failure), never by making a kernel hang; the
bounded wait itself giving up is covered by the wait self-test
(tests/test_gpu_exp2.py)."""

import pytest
import torch

import cache_gating_kv_b200 as fc
from tests.gpu_util import DEV

pytestmark = pytest.mark.gpu


def _gate_call(n_c=4, N=4096):
    x = torch.randn(n_c, N, device=DEV)
    v = torch.randn(n_c, N, device=DEV)
    dt = torch.full((n_c,), -0.1, device=DEV)
    st = torch.full((n_c,), 3, dtype=torch.int32, device=DEV)
    f = torch.zeros(n_c, device=DEV)
    l1 = torch.empty(n_c, device=DEV)
    mask = torch.empty(n_c, dtype=torch.uint8, device=DEV)
    ws = fc.workspace(fc.fc_gate_workspace_size(n_c, N))
    fc.fc_chunk_l1_gate(x, v, dt, st, 2, 0.05, f, l1, mask, ws)
    return ws, (x, v, dt, st, f, l1, mask)


def test_gate_word_clear_after_a_normal_call():
    ws, _ = _gate_call()
    assert fc.fc_check_workspace(fc.FC_WS_GATE, ws, 4)


def test_gate_planted_timeout_is_reported_and_cleared():
    n_c = 4
    ws, _ = _gate_call(n_c)
    ws.view(torch.int32)[n_c] = 1  # the word after the n_c completion counters
    assert not fc.fc_check_workspace(fc.FC_WS_GATE, ws, n_c)
    assert not fc.fc_check_workspace(fc.FC_WS_GATE, ws, n_c, clear=True)
    assert fc.fc_check_workspace(fc.FC_WS_GATE, ws, n_c)
    # the counters before it are untouched by the check
    assert int(ws.view(torch.int32)[:n_c].abs().sum().item()) == 0


def test_importance_planted_timeout():
    q = torch.randn(2, 256, 128, device=DEV).to(torch.bfloat16)
    k = torch.randn(2, 1024, 128, device=DEV).to(torch.bfloat16)
    imp = torch.empty(2, 1024, device=DEV)
    ws = fc.workspace(fc.fc_importance_workspace_size(fc.FC_BF16, 2, 256, 1024, 128))
    fc.fc_kv_importance(q, k, imp, ws)
    assert fc.fc_check_workspace(fc.FC_WS_IMPORTANCE, ws)
    ws.view(torch.int32)[0] = 7
    assert not fc.fc_check_workspace(fc.FC_WS_IMPORTANCE, ws, clear=True)
    assert fc.fc_check_workspace(fc.FC_WS_IMPORTANCE, ws)


def test_noalloc_gate_word_reads_the_static_scratch():
    n_c, N = 3, 8192
    x = torch.randn(n_c, N, device=DEV)
    v = torch.randn(n_c, N, device=DEV)
    dt = torch.full((n_c,), -0.1, device=DEV)
    st = torch.full((n_c,), 3, dtype=torch.int32, device=DEV)
    f = torch.zeros(n_c, device=DEV)
    l1 = torch.empty(n_c, device=DEV)
    mask = torch.empty(n_c, dtype=torch.uint8, device=DEV)
    fc.fc_chunk_l1_gate_noalloc(x, v, dt, st, 2, 0.05, f, l1, mask)
    assert fc.fc_check_workspace(fc.FC_WS_GATE_NOALLOC, None, n_c)


def test_gates_reject_overlapping_latents_before_launching():
    """x is updated in place while v is read (h_old overwritten while h_new is
    read): any overlap of the two [n][N] arrays is refused on the host, and
    nothing is written."""
    n_c, N = 3, 4096
    buf = torch.randn(n_c * N + 4, device=DEV)
    x = buf[:n_c * N].view(n_c, N)
    v_overlap = buf[4:].view(n_c, N)  # 16 bytes in: aligned, partly aliased
    before = buf.clone()
    dt = torch.full((n_c,), -0.1, device=DEV)
    st = torch.full((n_c,), 3, dtype=torch.int32, device=DEV)
    f = torch.zeros(n_c, device=DEV)
    l1 = torch.full((n_c,), -1.0, device=DEV)
    mask = torch.full((n_c,), 7, dtype=torch.uint8, device=DEV)
    ws = fc.workspace(fc.fc_gate_workspace_size(n_c, N))
    for call in (lambda: fc.fc_chunk_l1_gate(x, v_overlap, dt, st, 2, 0.05, f, l1, mask, ws),
                 lambda: fc.fc_chunk_l1_gate_noalloc(x, v_overlap, dt, st, 2, 0.05, f, l1, mask),
                 lambda: fc.fc_history_l1_gate(x, v_overlap, st, 2, 0.05, f, l1, mask, ws)):
        with pytest.raises(fc.FlowCacheError) as e:
            call()
        assert e.value.status == 1 and "overlap" in str(e.value)
    torch.cuda.synchronize()
    assert torch.equal(buf, before) and float(l1[0]) == -1.0 and int(mask[0]) == 7
