"""Plain CPU oracle for the FlowCache hot path.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline / reference legs of ``bench.py`` may
import or execute this module.  It shares no code with the CUDA path and never
imports it.

Source of every definition: the paper notes "Flow Caching for Autoregressive
Video Generation" (papernotes.org, ICLR 2026), section "方法详解 / 关键设计"
(method details / key designs):

* key design 1 -- relative L1 distance of chunk i at step t, inline equation
  ``L1_rel(X,t,i) = ||X^i_{t-1} - X^i_t||_1 / ||X^i_t||_1
                  = ||v(X^i_t,t,c) * dt||_1 / ||X^i_t||_1``;
* key design 2 -- the per-chunk recursive accumulator f: forced recompute
  (f = 0) for the first m steps, afterwards recompute and reset when
  ``f(X,t+1,i) + L1_rel(X,t,i) > eps``, else accumulate and reuse;
* key design 3 -- joint importance/redundancy KV-cache compression:
  importance = attention softmax of the denoising queries over the clean keys,
  averaged over queries, then 1D max-pooled; redundancy_j =
  softmax_j((1/L_k) sum_i S_ij) with S the cosine similarity of l2-normalised
  keys and a zeroed diagonal; Score = lam*Imp~ - (1-lam)*Red; keep the top-B
  tokens per head in the fixed B_budget buffer.

Arithmetic: float64 throughout, except where the method itself produces a
float32 tensor (the Euler update of the float32 latent, the float32 recurrence
state f, and the float32 score on which the top-B decision is taken: the
kernel's precision, so that both sides take every integer decision the same
way).  Matrix products and sorts are library calls (numpy); nothing is blocked
or fused beyond processing independent rows of a matrix a group at a time.

Readings of points the pages leave open:
the mask is the decision for the chunk's next forward; "first m steps" counts
per chunk; the comparison with eps is strict; ||X_t||_1 = 0 gives L1 = +inf
(or 0 when the update is also zero); a step counter < 0 marks an inactive
chunk that is left untouched; the importance softmax runs over the clean
candidate keys only with scale 1/sqrt(d); pooling is a stride-1 max filter
whose out-of-range taps are ignored; redundancy divides by L_k; a zero key
normalises to zero; top-B ties keep the lower token index and indices are
returned ascending; B >= L_k keeps every token and pads with -1.
"""

import math

import numpy as np

__all__ = [
    "gate_step",
    "history_gate_step",
    "gather_recompute",
    "scatter_velocity",
    "cache_commit",
    "cache_stream",
    "importance",
    "row_lse",
    "importance_at",
    "redundancy",
    "redundancy_logits_at",
    "maxpool1d",
    "score",
    "topb",
    "score_topb",
    "compact",
]

# Rows of a logits / similarity matrix that are formed at once.  Rows are
# independent, so the group size changes nothing but peak memory.
_ROWS = 256


# ---------------------------------------------------------------------------
# Chunkwise cache gate (key designs 1 and 2)
# ---------------------------------------------------------------------------
def gate_step(x, v, dt, step, m, eps, f):
    """One denoising step of the chunkwise cache gate, for every chunk.

    Follows key design 1 (relative L1 of the Euler update, its second form
    ``||v*dt||_1 / ||X_t||_1``) and key design 2 (the accumulator f).

    x    [n_c, N] float32  latent X_t (not modified; the update is returned)
    v    [n_c, N] float32  velocity applied at this step
    dt   [n_c]    float32  signed step of chunk c
    step [n_c]    int      steps chunk c has taken since it started; < 0 = inactive
    m    int               forced-recompute steps
    eps  float             threshold (compared in float32)
    f    [n_c]    float32  accumulator after the previous step

    Returns ``(x_next, f_next, l1, mask)``: float32 ``X_{t-1}``, float32 f,
    float32 L1_rel, uint8 recompute mask (1 = recompute at the next forward).
    """
    x = np.asarray(x, dtype=np.float32)
    v = np.asarray(v, dtype=np.float32)
    dt = np.asarray(dt, dtype=np.float32)
    step = np.asarray(step)
    f = np.asarray(f, dtype=np.float32)
    n_c = x.shape[0]
    eps32 = np.float32(eps)

    x_next = x.copy()
    f_next = f.copy()
    l1 = np.zeros(n_c, dtype=np.float32)
    mask = np.zeros(n_c, dtype=np.uint8)
    for c in range(n_c):
        if step[c] < 0:
            continue  # inactive chunk: nothing is touched
        update = v[c] * dt[c]  # v*dt, one float32 rounding
        x_next[c] = x[c] + update  # X_{t-1} = X_t + v*dt, one float32 rounding
        num = np.sum(np.abs(update.astype(np.float64)))
        den = np.sum(np.abs(x[c].astype(np.float64)))
        if den > 0.0:
            rel = num / den
        else:
            rel = math.inf if num > 0.0 else 0.0
        l1[c] = np.float32(rel)
        if step[c] < m:
            mask[c] = 1  # forced recompute, f = 0
            f_next[c] = np.float32(0.0)
        else:
            acc = np.float32(f[c] + l1[c])
            if acc > eps32:
                mask[c] = 1  # recompute and reset
                f_next[c] = np.float32(0.0)
            else:
                mask[c] = 0  # reuse and accumulate
                f_next[c] = acc
    return x_next, f_next, l1, mask


def history_gate_step(h_old, h_new, step, m, delta, f):
    """One step of the history-guided cache gate (a neighbouring method: the
    ARCache notes "Accelerating Autoregressive Video Diffusion via
    History-Guided Cache and Residual Correction", 关键设计 1, HGC).

    Delta = ||h_t - h_{t+1}||_1 / ||h_{t+1}||_1 (denominator at the older step
    h_{t+1}); the deviations are summed from the last refresh step t_ref down
    to t, and the step where the sum first exceeds delta refreshes:
    sum_{i=t+1}^{t_ref} Delta <= delta < sum_{i=t}^{t_ref} Delta.  The refresh
    step becomes t_ref, so its own Delta opens the next window (f = Delta after
    a refresh, where the FlowCache gate resets to 0).  The first m steps of a
    segment refresh unconditionally (same rule for f).

    h_old [n, N] float32 h_{t+1}; h_new [n, N] float32 h_t; step [n] (< 0:
    inactive, untouched); f [n] float32.  Returns (h_next = h_new copy for
    active segments, f_next, d_rel, refresh mask)."""
    h_old = np.asarray(h_old, dtype=np.float32)
    h_new = np.asarray(h_new, dtype=np.float32)
    step = np.asarray(step)
    f = np.asarray(f, dtype=np.float32)
    n = h_old.shape[0]
    delta32 = np.float32(delta)
    h_next = h_old.copy()
    f_next = f.copy()
    d = np.zeros(n, dtype=np.float32)
    mask = np.zeros(n, dtype=np.uint8)
    for c in range(n):
        if step[c] < 0:
            continue
        diff = h_new[c] - h_old[c]  # one float32 rounding
        num = np.sum(np.abs(diff.astype(np.float64)))
        den = np.sum(np.abs(h_old[c].astype(np.float64)))
        if den > 0.0:
            rel = num / den
        else:
            rel = math.inf if num > 0.0 else 0.0
        d[c] = np.float32(rel)
        h_next[c] = h_new[c]
        acc = np.float32(f[c] + d[c])
        if step[c] < m or acc > delta32:
            mask[c] = 1
            f_next[c] = d[c]  # the refresh step opens the next window
        else:
            mask[c] = 0
            f_next[c] = acc
    return h_next, f_next, d, mask


def gather_recompute(x, mask):
    """The chunks the gate marked for recompute (key design 2 and the
    flowchart: recompute chunks run the model forward, reuse chunks take their
    cached activations), gathered in chunk order into a dense batch.

    x [n_c, N], mask [n_c] uint8.  Returns (ids int32 [n_c] -- the recompute
    chunk indices ascending, then -1 --, count, dense [n_c, N]); only the first
    count rows of dense are part of the result."""
    x = np.asarray(x)
    n_c = x.shape[0]
    ids = np.full(n_c, -1, dtype=np.int32)
    sel = [c for c in range(n_c) if mask[c] != 0]
    ids[:len(sel)] = sel
    dense = np.zeros_like(x)
    for i, c in enumerate(sel):
        dense[i] = x[c]
    return ids, len(sel), dense


def scatter_velocity(v_cache, v_dense, ids, count):
    """Fresh velocities of the recomputed chunks back into the per-chunk cache:
    v_cache[ids[i]] = v_dense[i] for i < count; reused chunks keep theirs."""
    out = np.array(v_cache, copy=True)
    for i in range(count):
        out[ids[i]] = v_dense[i]
    return out


# ---------------------------------------------------------------------------
# Importance (key design 3)
# ---------------------------------------------------------------------------
def _scale(d, scale):
    return 1.0 / math.sqrt(d) if (scale is None or scale <= 0) else float(scale)


def importance(q, k, scale=None):
    """Pre-pooling importance ``Imp[h, j] = (1/L_q) sum_q softmax_j(q.k_j*scale)``.

    Key design 3: the attention softmax of the current denoising queries over
    the clean keys, averaged over the queries.  q [H, L_q, d], k [H, L_k, d];
    returns float64 [H, L_k].  Each logits row is formed in full and put
    through a max-subtracted softmax.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    H, Lq, d = q.shape
    Lk = k.shape[1]
    c = _scale(d, scale)
    imp = np.zeros((H, Lk), dtype=np.float64)
    for h in range(H):
        for q0 in range(0, Lq, _ROWS):
            s = c * (q[h, q0:q0 + _ROWS] @ k[h].T)  # logits rows
            s -= s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)  # softmax over the L_k keys
            imp[h] += p.sum(axis=0)
        imp[h] /= Lq
    return imp


def row_lse(q, k, scale=None):
    """``log sum_j exp(q.k_j*scale)`` for every query row (the softmax's log
    normaliser in key design 3).  Returns float64 [H, L_q]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    H, Lq, d = q.shape
    c = _scale(d, scale)
    out = np.empty((H, Lq), dtype=np.float64)
    for h in range(H):
        for q0 in range(0, Lq, _ROWS):
            s = c * (q[h, q0:q0 + _ROWS] @ k[h].T)
            mx = s.max(axis=1)
            out[h, q0:q0 + _ROWS] = mx + np.log(np.exp(s - mx[:, None]).sum(axis=1))
    return out


def importance_at(q, k, heads, cols, lse, scale=None):
    """``Imp[h, j]`` at chosen (head, key) pairs, given the row normalisers
    ``lse`` of :func:`row_lse`: ``(1/L_q) sum_q exp(q.k_j*scale - lse_q)``.

    The same definition as :func:`importance`, evaluated one output at a
    time, for checks at sizes where the full table is too slow."""
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[2]
    c = _scale(d, scale)
    out = np.empty(len(cols), dtype=np.float64)
    for n, (h, j) in enumerate(zip(heads, cols)):
        kj = np.asarray(k[h, j], dtype=np.float64)
        s = c * (q[h] @ kj)
        out[n] = np.exp(s - lse[h]).mean()
    return out


# ---------------------------------------------------------------------------
# Redundancy (key design 3)
# ---------------------------------------------------------------------------
def _unit_rows(k):
    norms = np.sqrt((k * k).sum(axis=-1, keepdims=True))
    return k / np.maximum(norms, 1e-12)  # a zero key stays zero


def redundancy(k):
    """``Red[h, j] = softmax_j((1/L_k) sum_i S_ij)`` with ``S`` the cosine
    similarity of l2-normalised keys and ``S_jj = 0`` (key design 3).

    Forms every row of the L_k x L_k similarity matrix (brute force; no
    algebraic shortcut).  k [H, L_k, d]; returns float64 [H, L_k]."""
    k = np.asarray(k, dtype=np.float64)
    H, Lk, _ = k.shape
    red = np.empty((H, Lk), dtype=np.float64)
    for h in range(H):
        kh = _unit_rows(k[h])
        col = np.zeros(Lk, dtype=np.float64)
        for i0 in range(0, Lk, _ROWS):
            S = kh[i0:i0 + _ROWS] @ kh.T  # rows i0.. of the cosine matrix
            rows = np.arange(i0, min(i0 + _ROWS, Lk))
            S[rows - i0, rows] = 0.0  # zero the diagonal
            col += S.sum(axis=0)
        r = col / Lk
        e = np.exp(r - r.max())
        red[h] = e / e.sum()
    return red


def redundancy_logits_at(k, heads, cols):
    """``r[h, j] = (1/L_k) sum_{i != j} khat_i . khat_j`` at chosen pairs: the
    softmax argument of the redundancy, one column at a time (brute force)."""
    out = np.empty(len(cols), dtype=np.float64)
    for n, (h, j) in enumerate(zip(heads, cols)):
        kh = _unit_rows(np.asarray(k[h], dtype=np.float64))
        s = kh @ kh[j]
        s[j] = 0.0
        out[n] = s.sum() / kh.shape[0]
    return out


# ---------------------------------------------------------------------------
# Pooling, score, top-B, compaction (key design 3)
# ---------------------------------------------------------------------------
def maxpool1d(x, window):
    """Stride-1 max filter of odd width ``window`` along the last axis; taps
    that fall outside the sequence are ignored (output length = input length)."""
    x = np.asarray(x)
    L = x.shape[-1]
    r = window // 2
    out = np.empty_like(x)
    for j in range(L):
        out[..., j] = x[..., max(0, j - r):min(L, j + r + 1)].max(axis=-1)
    return out


def score(imp, red, lam, window):
    """``Score = lam*Imp~ - (1-lam)*Red`` with ``Imp~`` the max-pooled
    importance, evaluated in float32 as ``fl(fl(lam*Imp~) - fl(fl(1-lam)*Red))``.

    float32 is the precision in which the selection is decided on both sides.
    imp, red [H, L_k] (rounded to float32 first); returns float32 [H, L_k]."""
    imp32 = np.asarray(imp, dtype=np.float32)
    red32 = np.asarray(red, dtype=np.float32)
    lam32 = np.float32(lam)
    one_minus = np.float32(np.float32(1.0) - lam32)
    pooled = maxpool1d(imp32, window)
    a = (lam32 * pooled).astype(np.float32)
    b = (one_minus * red32).astype(np.float32)
    return (a - b).astype(np.float32)


def topb(sc, B):
    """Per-head indices of the B largest scores; equal scores keep the lower
    token index; indices returned ascending.  ``B >= L_k`` keeps every token
    and pads the rest of the row with -1.  sc [H, L_k]; returns int32 [H, B]."""
    sc = np.asarray(sc)
    H, Lk = sc.shape
    out = np.full((H, B), -1, dtype=np.int32)
    pos = np.arange(Lk)
    for h in range(H):
        order = np.lexsort((pos, -sc[h].astype(np.float64)))  # score desc, index asc
        keep = np.sort(order[:min(B, Lk)])
        out[h, :keep.size] = keep
    return out


def score_topb(imp, red, lam, window, B):
    """Score then top-B: returns ``(score float32 [H, L_k], idx int32 [H, B])``."""
    sc = score(imp, red, lam, window)
    return sc, topb(sc, B)


def compact(k, v, idx):
    """``K_out[h, r] = K[h, idx[h, r]]`` and the same for V; rows whose index
    is -1 are zero.  Returns new arrays of shape [H, B, d]."""
    k = np.asarray(k)
    v = np.asarray(v)
    H, B = idx.shape
    d = k.shape[2]
    k_out = np.zeros((H, B, d), dtype=k.dtype)
    v_out = np.zeros((H, B, d), dtype=v.dtype)
    for h in range(H):
        for r in range(B):
            j = idx[h, r]
            if j >= 0:
                k_out[h, r] = k[h, j]
                v_out[h, r] = v[h, j]
    return k_out, v_out


# ---------------------------------------------------------------------------
# Cache buffer management around compression (key design 3 and the flowchart:
# a finished chunk enters the KV cache; when the reserved cache is full it is
# merged into the candidates and each head keeps its top-B tokens)
# ---------------------------------------------------------------------------

def cache_commit(k_buf, v_buf, n_clean, C, B_budget, q, lam, window, scale=None):
    """One finished chunk enters the fixed buffer ``B_total = B_budget + C``.

    k_buf, v_buf [H, B_budget + C, d]: rows [0, n_clean) hold the compressed
    clean tokens, rows [n_clean, n_clean + C) the chunk that has just finished
    denoising.  q [H, L_q, d] are the queries of the chunk now denoising.

    If the n_clean + C candidates fit in B_budget they are kept as they are:
    returns (k_buf, v_buf, n_clean + C, None).  Otherwise the candidates are
    scored (importance of q over them, redundancy, joint score) and every head
    keeps its top-B_budget; returns (k_next, v_next, B_budget, idx) with the
    kept rows in rows [0, B_budget) of new buffers of the same shape, the rest
    zero, and idx [H, B_budget] the kept candidate rows."""
    H, cap, d = k_buf.shape
    assert cap == B_budget + C and 0 <= n_clean <= B_budget
    L = n_clean + C
    if L <= B_budget:
        return k_buf, v_buf, L, None
    kc, vc = k_buf[:, :L], v_buf[:, :L]
    imp = importance(q, kc, scale)
    red = redundancy(kc)
    _, idx = score_topb(imp, red, lam, window, B_budget)
    ko, vo = compact(kc, vc, idx)
    k_next = np.zeros_like(k_buf)
    v_next = np.zeros_like(v_buf)
    k_next[:, :B_budget] = ko
    v_next[:, :B_budget] = vo
    return k_next, v_next, B_budget, idx


def cache_stream(chunks_k, chunks_v, queries, B_budget, lam, window, scale=None):
    """Chunks finish one after another: chunk i's K/V [H, C, d] go into the
    active rows, then ``cache_commit`` with queries[i].  Returns the final
    (k_buf, v_buf, n_clean) and the clean length after each chunk."""
    H, C, d = chunks_k[0].shape
    k_buf = np.zeros((H, B_budget + C, d), dtype=chunks_k[0].dtype)
    v_buf = np.zeros_like(k_buf)
    n = 0
    lengths = []
    for kc, vc, q in zip(chunks_k, chunks_v, queries):
        k_buf = k_buf.copy()
        v_buf = v_buf.copy()
        k_buf[:, n:n + C] = kc
        v_buf[:, n:n + C] = vc
        k_buf, v_buf, n, _ = cache_commit(k_buf, v_buf, n, C, B_budget, q, lam, window, scale)
        lengths.append(n)
    return k_buf, v_buf, n, lengths

