"""The C-ABI boundary on the host: the library loads, exports every call that
include/*.h declares, and rejects bad arguments before launching anything.
No test here needs a GPU (no compute call reaches a kernel)."""

import ctypes
import glob
import os
import re

import pytest

import cache_gating_kv_b200 as fc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DECL = re.compile(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(fc_\w+)\s*\(", re.M)


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        names.update(DECL.findall(open(h).read()))
    return sorted(names)


def test_header_declares_the_calls():
    names = _declared()
    for n in ["fc_chunk_l1_gate", "fc_kv_importance", "fc_kv_redundancy", "fc_kv_score_topb",
              "fc_kv_compact", "fc_last_error"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(fc.library_path)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_version_and_workspace_queries():
    lib = fc.library()
    assert lib.fc_version() >= 100
    assert lib.fc_gate_workspace_size(4, 777600) > 0
    assert lib.fc_gate_workspace_size(0, 10) == 0
    assert lib.fc_importance_workspace_size(fc.FC_BF16, 24, 4096, 16384, 128) >= 24 * 4096 * 4
    assert lib.fc_redundancy_workspace_size(fc.FC_BF16, 24, 16384, 128) > 0
    assert lib.fc_redundancy_workspace_size(fc.FC_BF16, 24, 16384, 96) == 0
    assert lib.fc_score_topb_workspace_size(24, 16384, 8192) >= 24 * 16384 * 4


NULL = None


def test_gate_rejects_bad_sizes_before_touching_memory():
    lib = fc.library()
    args = lambda n_c, N, m, ws_bytes: lib.fc_chunk_l1_gate(  # noqa: E731
        NULL, NULL, n_c, N, NULL, NULL, m, 0.1, NULL, NULL, NULL, NULL, ws_bytes, NULL)
    assert args(0, 10, 1, 1 << 20) == 1
    assert args(70000, 10, 1, 1 << 30) == 1
    assert args(2, -1, 1, 1 << 20) == 1
    assert args(2, 10, -1, 1 << 20) == 1
    assert args(2, 10, 1, 1 << 20) == 3  # ws is NULL -> workspace error
    assert b"workspace" in lib.fc_last_error()


def test_gate_rejects_null_tensor_with_message():
    lib = fc.library()
    ws = ctypes.create_string_buffer(1 << 20)
    buf = ctypes.addressof(ws)
    st = lib.fc_chunk_l1_gate(NULL, NULL, 2, 10, NULL, NULL, 1, 0.1, NULL, NULL, NULL, buf,
                              1 << 20, NULL)
    assert st == 1 and lib.fc_last_error() == b"x is NULL"


def test_host_pointer_is_rejected():
    """A host pointer never reaches a kernel: without a GPU the pointer query
    fails (FC_ERR_CUDA); with one, host memory is FC_ERR_INVALID_ARG."""
    lib = fc.library()
    host = ctypes.create_string_buffer(1 << 16)
    p = (ctypes.addressof(host) + 15) // 16 * 16
    st = lib.fc_kv_compact(p, p, fc.FC_BF16, 1, 8, 128, p, 4, p + 4096, p + 8192, NULL)
    assert st in (1, 4)
    assert lib.fc_last_error() != b""


def test_kv_calls_reject_bad_shapes():
    lib = fc.library()
    # d not in {64, 128}
    assert lib.fc_kv_importance(NULL, NULL, fc.FC_BF16, 2, 8, 8, 96, 0.0, NULL, NULL, 0, NULL) == 2
    assert lib.fc_kv_redundancy(NULL, fc.FC_BF16, 2, 8, 32, NULL, NULL, 0, NULL) == 2
    # empty sizes
    assert lib.fc_kv_importance(NULL, NULL, fc.FC_BF16, 0, 8, 8, 64, 0.0, NULL, NULL, 0, NULL) == 1
    assert lib.fc_kv_importance(NULL, NULL, fc.FC_BF16, 2, 0, 8, 64, 0.0, NULL, NULL, 0, NULL) == 1
    # unknown dtype
    assert lib.fc_kv_redundancy(NULL, 7, 2, 8, 64, NULL, NULL, 0, NULL) == 1
    # more keys than the redundancy's fixed-point sums serve (2^26)
    assert lib.fc_kv_redundancy(NULL, fc.FC_BF16, 1, (1 << 26) + 1, 64, NULL, NULL, 0, NULL) == 2
    assert b"2^26" in lib.fc_last_error() or b"67108864" in lib.fc_last_error()
    # workspace too small
    assert lib.fc_kv_importance(NULL, NULL, fc.FC_BF16, 2, 8, 8, 64, 0.0, NULL, NULL, 4, NULL) == 3
    # score/top-B: B < 1, even or too wide pool window
    assert lib.fc_kv_score_topb(NULL, NULL, 2, 8, 7, 0.5, 0, NULL, NULL, NULL, 1 << 20, NULL) == 1
    assert lib.fc_kv_score_topb(NULL, NULL, 2, 8, 6, 0.5, 4, NULL, NULL, NULL, 1 << 20, NULL) == 1
    assert lib.fc_kv_score_topb(NULL, NULL, 2, 8, 513, 0.5, 4, NULL, NULL, NULL, 1 << 20,
                                NULL) == 1
    assert lib.fc_kv_compact(NULL, NULL, fc.FC_BF16, 2, 8, 64, NULL, 0, NULL, NULL, NULL) == 1
    assert lib.fc_kv_compact(NULL, NULL, fc.FC_BF16, 2, 8, 64, NULL, 4, NULL, NULL, NULL) == 1


def test_binding_fails_loudly_without_cuda_tensors():
    import torch
    x = torch.zeros(2, 8)
    with pytest.raises(fc.FlowCacheError):
        fc.fc_kv_redundancy(x.view(1, 2, 8), torch.zeros(1, 2), torch.zeros(256, dtype=torch.uint8))


def test_product_package_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "cache_gating_kv_b200")
    for path in glob.glob(os.path.join(pkg, "**", "*.py"), recursive=True) + \
            glob.glob(os.path.join(pkg, "csrc", "*")):
        src = open(path, errors="replace").read()
        assert not re.search(r"^\s*(import|from)\s+oracle\b", src, re.M), path
        assert "flowcache_oracle" not in src, path


def test_selftest_entries_validate_on_the_host():
    import ctypes as C
    lib = fc.library()
    lib.fc_selftest_wait_timeout.restype = C.c_int
    lib.fc_selftest_wait_timeout.argtypes = [C.c_longlong, C.c_void_p, C.c_void_p]
    assert lib.fc_selftest_wait_timeout(-1, None, None) == 1
    assert lib.fc_selftest_wait_timeout(10**10, None, None) == 1
    assert lib.fc_selftest_wait_timeout(1000, None, None) == 1  # NULL error word
    lib.fc_selftest_exp2.restype = C.c_int
    lib.fc_selftest_exp2.argtypes = [C.c_void_p] * 3 + [C.c_int, C.c_void_p]
    assert lib.fc_selftest_exp2(None, None, None, 3, None) == 1  # odd n


def test_mask_consumer_validates_on_the_host():
    lib = fc.library()
    # n_chunks out of range
    assert lib.fc_gather_recompute(NULL, NULL, 0, 8, NULL, NULL, NULL, NULL) == 1
    assert lib.fc_gather_recompute(NULL, NULL, 70000, 8, NULL, NULL, NULL, NULL) == 1
    assert lib.fc_scatter_velocity(NULL, NULL, NULL, 0, 8, NULL, NULL) == 1
    # negative size, NULL buffers
    assert lib.fc_gather_recompute(NULL, NULL, 4, -1, NULL, NULL, NULL, NULL) == 1
    assert lib.fc_gather_recompute(NULL, NULL, 4, 8, NULL, NULL, NULL, NULL) == 1
    assert lib.fc_last_error() == b"x is NULL"
    assert lib.fc_scatter_velocity(NULL, NULL, NULL, 4, 8, NULL, NULL) == 1
    assert lib.fc_last_error() == b"v_dense is NULL"


def test_cache_commit_validates_and_keeps_fitting_chunks_on_the_host():
    lib = fc.library()
    n_next, comp = ctypes.c_int(-1), ctypes.c_int(-1)
    ref = (ctypes.byref(n_next), ctypes.byref(comp))

    host = ctypes.create_string_buffer(256)

    def commit(dtype=fc.FC_BF16, H=2, Lq=8, d=64, B=96, C=32, n=0, pool=3, ws_bytes=0):
        ws = ctypes.addressof(host) if ws_bytes else NULL
        return lib.fc_kv_cache_commit(NULL, NULL, NULL, NULL, NULL, dtype, H, Lq, d, B, C, n,
                                      0.0, pool, 0.5, NULL, ws, ws_bytes, *ref, NULL)

    # the chunk fits: nothing is launched and no device pointer is needed
    assert commit(n=64) == 0 and (n_next.value, comp.value) == (96, 0)
    assert lib.fc_last_launches() == 0
    n_next.value = comp.value = -1
    assert commit(B=96, C=96, n=0) == 0 and (n_next.value, comp.value) == (96, 0)
    # any chunk size: B_budget need not be a multiple of C, n_clean any count
    n_next.value = comp.value = -1
    assert commit(B=100, C=32, n=68) == 0 and (n_next.value, comp.value) == (100, 0)
    assert commit(n=16) == 0 and (n_next.value, comp.value) == (48, 0)
    assert lib.fc_last_launches() == 0
    # d unsupported
    assert commit(d=96) == 2
    # n_clean out of range, C < 1, C > B_budget, even window
    assert commit(n=-1) == 1
    assert commit(n=128) == 1
    assert commit(C=0) == 1
    assert commit(C=128) == 1
    assert commit(n=64, pool=4) == 1
    # a full cache needs the workspace
    assert commit(n=96) == 3
    assert b"workspace" in lib.fc_last_error()
    # the error paths leave the outputs alone
    n_next.value = comp.value = -1
    assert commit(n=96, ws_bytes=1 << 30) == 1  # then the NULL q (ws is never read here)
    assert lib.fc_last_error() == b"q is NULL"
    assert (n_next.value, comp.value) == (-1, -1)
    assert lib.fc_kv_cache_workspace_size(fc.FC_BF16, 2, 8, 96, 32, 64) > 0
    assert lib.fc_kv_cache_workspace_size(fc.FC_BF16, 2, 8, 96, 32, 96) == 0


def test_check_workspace_validates_on_the_host():
    lib = fc.library()
    assert lib.fc_check_workspace(9, NULL, 1, 0, NULL) == 1  # unknown kind
    assert lib.fc_check_workspace(fc.FC_WS_GATE, NULL, 0, 0, NULL) == 1  # n_chunks < 1
    assert lib.fc_check_workspace(fc.FC_WS_GATE, NULL, 4, 0, NULL) == 1
    assert lib.fc_last_error() == b"ws is NULL"
    assert lib.fc_check_workspace(fc.FC_WS_IMPORTANCE, NULL, 0, 0, NULL) == 1
    assert lib.fc_check_workspace(fc.FC_WS_GATE_NOALLOC, NULL, 33, 0, NULL) == 1  # > 32 chunks
