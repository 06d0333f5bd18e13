"""FlowCache hot path on B200: thin Python binding of ``libflowcache.so``.

Every function here marshals torch CUDA tensors into the C-ABI call of the
same name declared in ``include/flowcache.h``; all arithmetic runs in the
library's CUDA kernels.  There is no CPU fallback: if the shared library is
missing or fails to load, every call raises :class:`FlowCacheError`.

Method: "Flow Caching for Autoregressive Video Generation" (papernotes.org),
方法详解 / 关键设计 1-3 (chunkwise relative-L1 cache gate; joint
importance-redundancy KV-cache compression).
"""

import ctypes
import os

import torch

__all__ = [
    "FlowCacheError",
    "FC_F32",
    "FC_BF16",
    "library",
    "library_path",
    "fc_version",
    "fc_last_launches",
    "fc_chunk_l1_gate",
    "fc_chunk_l1_gate_noalloc",
    "fc_history_l1_gate",
    "fc_gather_recompute",
    "fc_scatter_velocity",
    "fc_kv_cache_workspace_size",
    "fc_check_workspace",
    "FC_WS_GATE",
    "FC_WS_GATE_NOALLOC",
    "FC_WS_IMPORTANCE",
    "FC_WS_CACHE",
    "fc_kv_cache_commit",
    "fc_kv_importance",
    "fc_kv_redundancy",
    "fc_kv_score_topb",
    "fc_kv_compact",
    "fc_gate_workspace_size",
    "fc_importance_workspace_size",
    "fc_redundancy_workspace_size",
    "fc_score_topb_workspace_size",
    "workspace",
]

FC_F32, FC_BF16 = 0, 1
_STATUS = {0: "FC_OK", 1: "FC_ERR_INVALID_ARG", 2: "FC_ERR_UNSUPPORTED", 3: "FC_ERR_WORKSPACE",
           4: "FC_ERR_CUDA", 5: "FC_ERR_TIMEOUT"}

library_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libflowcache.so")
_lib = None


class FlowCacheError(RuntimeError):
    """A libflowcache call returned an error status, or the library is missing."""

    def __init__(self, msg, status=None):
        super().__init__(msg)
        self.status = status


def _declare(lib):
    c_int, c_i64, c_f, c_sz, c_p = (ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t,
                                     ctypes.c_void_p)
    sig = {
        "fc_last_error": (ctypes.c_char_p, []),
        "fc_version": (c_int, []),
        "fc_last_launches": (c_int, []),
        "fc_gate_workspace_size": (c_sz, [c_int, c_i64]),
        "fc_chunk_l1_gate": (c_int, [c_p, c_p, c_int, c_i64, c_p, c_p, ctypes.c_int32, c_f, c_p,
                                     c_p, c_p, c_p, c_sz, c_p]),
        "fc_chunk_l1_gate_noalloc": (c_int, [c_p, c_p, c_int, c_i64, c_p, c_p, ctypes.c_int32,
                                             c_f, c_p, c_p, c_p, c_p]),
        "fc_history_l1_gate": (c_int, [c_p, c_p, c_int, c_i64, c_p, ctypes.c_int32, c_f, c_p, c_p,
                                       c_p, c_p, c_sz, c_p]),
        "fc_gather_recompute": (c_int, [c_p, c_p, c_int, c_i64, c_p, c_p, c_p, c_p]),
        "fc_scatter_velocity": (c_int, [c_p, c_p, c_p, c_int, c_i64, c_p, c_p]),
        "fc_importance_workspace_size": (c_sz, [c_int, c_int, c_int, c_int, c_int]),
        "fc_kv_importance": (c_int, [c_p, c_p, c_int, c_int, c_int, c_int, c_int, c_f, c_p, c_p,
                                     c_sz, c_p]),
        "fc_redundancy_workspace_size": (c_sz, [c_int, c_int, c_int, c_int]),
        "fc_kv_redundancy": (c_int, [c_p, c_int, c_int, c_int, c_int, c_p, c_p, c_sz, c_p]),
        "fc_score_topb_workspace_size": (c_sz, [c_int, c_int, c_int]),
        "fc_kv_score_topb": (c_int, [c_p, c_p, c_int, c_int, c_int, c_f, c_int, c_p, c_p, c_p,
                                     c_sz, c_p]),
        "fc_kv_compact": (c_int, [c_p, c_p, c_int, c_int, c_int, c_int, c_p, c_int, c_p, c_p,
                                  c_p]),
        "fc_kv_cache_workspace_size": (c_sz, [c_int, c_int, c_int, c_int, c_int, c_int]),
        "fc_check_workspace": (c_int, [c_int, c_p, c_int, c_int, c_p]),
        "fc_kv_cache_commit": (c_int, [c_p, c_p, c_p, c_p, c_p, c_int, c_int, c_int, c_int, c_int,
                                       c_int, c_int, c_f, c_int, c_f, c_p, c_p, c_sz,
                                       ctypes.POINTER(c_int), ctypes.POINTER(c_int), c_p]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def library():
    """The loaded ``ctypes.CDLL`` (loaded on first use)."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise FlowCacheError(
                f"{library_path} is not built; run `python -m cache_gating_kv_b200.build`")
        try:
            _lib = _declare(ctypes.CDLL(library_path))
        except OSError as e:
            raise FlowCacheError(f"cannot load {library_path}: {e}") from e
    return _lib


def _check(name, st):
    if st != 0:
        msg = library().fc_last_error().decode(errors="replace")
        raise FlowCacheError(f"{name}: {_STATUS.get(st, st)}: {msg}", st)


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise FlowCacheError("tensor arguments must be CUDA tensors")
    if not t.is_contiguous():
        raise FlowCacheError("tensor arguments must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return FC_BF16
    if t.dtype == torch.float32:
        return FC_F32
    raise FlowCacheError(f"unsupported dtype {t.dtype}")


def fc_version():
    return library().fc_version()


def fc_last_launches():
    """Kernel launches (memsets included) the last compute call on this thread
    enqueued."""
    return library().fc_last_launches()


# ---- workspace sizes and allocation ----------------------------------------
def fc_gate_workspace_size(n_chunks, n_per_chunk):
    return library().fc_gate_workspace_size(n_chunks, n_per_chunk)


def fc_importance_workspace_size(dtype, H, Lq, Lk, d):
    return library().fc_importance_workspace_size(dtype, H, Lq, Lk, d)


def fc_redundancy_workspace_size(dtype, H, Lk, d):
    return library().fc_redundancy_workspace_size(dtype, H, Lk, d)


def fc_score_topb_workspace_size(H, Lk, B):
    return library().fc_score_topb_workspace_size(H, Lk, B)


def fc_kv_cache_workspace_size(dtype, H, Lq, B_budget, C, d):
    return library().fc_kv_cache_workspace_size(dtype, H, Lq, B_budget, C, d)


FC_WS_GATE, FC_WS_GATE_NOALLOC, FC_WS_IMPORTANCE, FC_WS_CACHE = 0, 1, 2, 3


def fc_check_workspace(kind, ws=None, n_chunks=0, clear=False, stream=None):
    """True if no bounded device-side wait of the calls that used ``ws`` gave
    up (synchronises the stream); False if one did (their outputs are not
    valid).  ``clear`` resets the error word after reading it."""
    st = library().fc_check_workspace(int(kind), _p(ws), int(n_chunks), 1 if clear else 0,
                                      _s(stream))
    if st == 5:
        return False
    _check("fc_check_workspace", st)
    return True


def workspace(nbytes, device=None):
    """A zero-filled device byte buffer of ``nbytes`` (at least 256) bytes."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


# ---- the five calls -----------------------------------------------------------
def fc_chunk_l1_gate(x, v, dt, step, m, eps, f, l1_rel, recompute, ws, stream=None):
    """Chunkwise cache gate step (in place on ``x`` and ``f``).  x, v: [n_c, N]
    float32; dt: [n_c] float32; step: [n_c] int32; f, l1_rel: [n_c] float32;
    recompute: [n_c] uint8; ws from :func:`fc_gate_workspace_size` (zeroed once)."""
    n_c, N = x.shape
    st = library().fc_chunk_l1_gate(_p(x), _p(v), n_c, N, _p(dt), _p(step), int(m), float(eps),
                                     _p(f), _p(l1_rel), _p(recompute), _p(ws), ws.numel(),
                                     _s(stream))
    _check("fc_chunk_l1_gate", st)


def fc_history_l1_gate(h_old, h_new, step, m, delta, f, d_rel, refresh, ws, stream=None):
    """History-guided gate step (in place on ``h_old`` and ``f``): h_old is
    h_{t+1} in and h_t out.  [n, N] float32 snapshots; step [n] int32; f, d_rel
    [n] float32; refresh [n] uint8; ws from :func:`fc_gate_workspace_size`."""
    n, N = h_old.shape
    st = library().fc_history_l1_gate(_p(h_old), _p(h_new), n, N, _p(step), int(m), float(delta),
                                       _p(f), _p(d_rel), _p(refresh), _p(ws), ws.numel(),
                                       _s(stream))
    _check("fc_history_l1_gate", st)


def fc_chunk_l1_gate_noalloc(x, v, dt, step, m, eps, f, l1_rel, recompute, stream=None):
    """The gate step without a workspace, for callers that cannot allocate
    device memory while they run it (the library keeps a fixed static scratch
    array instead).  At most 32 chunks per call; calls must not overlap on the
    GPU; the first call on a device should precede any stream capture."""
    n_c, N = x.shape
    st = library().fc_chunk_l1_gate_noalloc(_p(x), _p(v), n_c, N, _p(dt), _p(step), int(m),
                                             float(eps), _p(f), _p(l1_rel), _p(recompute),
                                             _s(stream))
    _check("fc_chunk_l1_gate_noalloc", st)


def fc_gather_recompute(x, recompute, dense, ids, count, stream=None):
    """Gather the recompute chunks' rows of x [n_c, N] into dense [n_c, N];
    ids [n_c] int32 and count [1] int32 are written on the device."""
    n_c, N = x.shape
    st = library().fc_gather_recompute(_p(x), _p(recompute), n_c, N, _p(dense), _p(ids),
                                        _p(count), _s(stream))
    _check("fc_gather_recompute", st)


def fc_scatter_velocity(v_dense, ids, count, v_cache, stream=None):
    """v_cache[ids[i]] = v_dense[i] for i < count (device-side count)."""
    n_c, N = v_cache.shape
    st = library().fc_scatter_velocity(_p(v_dense), _p(ids), _p(count), n_c, N, _p(v_cache),
                                        _s(stream))
    _check("fc_scatter_velocity", st)


def fc_kv_importance(q, k, imp, ws, scale=0.0, stream=None):
    """Pre-pooling importance.  q [H, Lq, d], k [H, Lk, d] (bf16 or float32);
    imp [H, Lk] float32 out."""
    H, Lq, d = q.shape
    Lk = k.shape[1]
    st = library().fc_kv_importance(_p(q), _p(k), _dtype_code(q), H, Lq, Lk, d, float(scale),
                                     _p(imp), _p(ws), ws.numel(), _s(stream))
    _check("fc_kv_importance", st)


def fc_kv_redundancy(k, red, ws, stream=None):
    """Redundancy.  k [H, Lk, d]; red [H, Lk] float32 out."""
    H, Lk, d = k.shape
    st = library().fc_kv_redundancy(_p(k), _dtype_code(k), H, Lk, d, _p(red), _p(ws), ws.numel(),
                                     _s(stream))
    _check("fc_kv_redundancy", st)


def fc_kv_score_topb(imp, red, pool_window, lam, B, idx, ws, score=None, stream=None):
    """Pooled joint score and per-head top-B.  imp, red [H, Lk] float32;
    idx [H, B] int32 out (ascending); score [H, Lk] float32 out or None."""
    H, Lk = imp.shape
    st = library().fc_kv_score_topb(_p(imp), _p(red), H, Lk, int(pool_window), float(lam), int(B),
                                     _p(score), _p(idx), _p(ws), ws.numel(), _s(stream))
    _check("fc_kv_score_topb", st)


def fc_kv_cache_commit(q, k_buf, v_buf, k_next, v_next, n_clean, C, ws, pool_window, lam,
                       scale=0.0, idx=None, stream=None):
    """One finished chunk enters the cache buffer [H, B_budget + C, d]; returns
    (n_next, compressed).  When compressed, the kept rows are in rows
    [0, B_budget) of k_next / v_next and the caller swaps the buffers."""
    H, cap, d = k_buf.shape
    Lq = q.shape[1]
    n_next, comp = ctypes.c_int(-1), ctypes.c_int(-1)
    st = library().fc_kv_cache_commit(
        _p(q), _p(k_buf), _p(v_buf), _p(k_next), _p(v_next), _dtype_code(k_buf), H, Lq, d,
        cap - C, C, n_clean, float(scale), int(pool_window), float(lam), _p(idx), _p(ws),
        0 if ws is None else ws.numel() * ws.element_size(), ctypes.byref(n_next), ctypes.byref(comp), _s(stream))
    _check("fc_kv_cache_commit", st)
    return n_next.value, bool(comp.value)


def fc_kv_compact(k, v, idx, k_out, v_out, stream=None):
    """Gather the kept rows: k_out[h, r] = k[h, idx[h, r]] (and V)."""
    H, Lk, d = k.shape
    B = idx.shape[1]
    st = library().fc_kv_compact(_p(k), _p(v), _dtype_code(k), H, Lk, d, _p(idx), B, _p(k_out),
                                  _p(v_out), _s(stream))
    _check("fc_kv_compact", st)
