"""Seeded synthetic workloads for the FlowCache hot path.

This module only draws inputs.  It holds none of the method's arithmetic (no
L1 distance, no accumulator, no softmax, no score), so the CUDA path and the
CPU oracle can both consume its output without sharing any of the method.

Shapes follow the settings of "Flow Caching for Autoregressive Video
Generation" (papernotes.org): the gate hyper-parameters m and eps of key
design 2 (MAGI-1 m=5, eps 0.01 slow / 0.015 fast; SkyReels-V2 m=4, eps 0.1 /
0.15) and the per-head compression of key design 3.  The pages describe no
dataset for these tensors, so keys follow AR(1) random walks along the token
axis (plus duplicate structure), queries and values are standard normal, and
the gate latents follow a single-point flow-matching toy with the power-law
schedule sigma(t) = (t/T)^p of Theorem 1.

Random streams: numpy PCG64 generators keyed by (seed, role, layer, head), so
that any head of any layer can be drawn on its own.  bf16 workloads round Q, K
and V to bfloat16 once; both sides consume those rounded values.
"""

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from typing import Optional, Sequence, Tuple

import numpy as np
import scipy.signal
import torch

__all__ = [
    "KVConfig",
    "GateConfig",
    "KV_CONFIGS",
    "CacheConfig",
    "CACHE_CONFIGS",
    "cache_inputs",
    "GATE_CONFIGS",
    "kv_inputs",
    "kv_head",
    "gate_initial",
    "gate_velocity",
    "gate_dt",
    "gate_step_counters",
]

_ROLE_Q, _ROLE_K, _ROLE_V, _ROLE_DUP, _ROLE_LOWRANK = 1, 2, 3, 4, 5
_ROLE_GATE_X0, _ROLE_GATE_NOISE, _ROLE_GATE_V = 11, 12, 13


@dataclass(frozen=True)
class KVConfig:
    """One compression workload (per layer: H heads of L_q queries and L_k keys)."""

    name: str
    H: int
    d: int
    Lq: int
    Lk: int
    B: int
    lam: Tuple[float, ...]
    pool: int
    dtype: str  # "f32" or "bf16"
    rho: float
    noise: Optional[float] = None  # AR innovation coefficient; default sqrt(1-rho^2)
    structure: str = "ar"  # "ar", "near_dup_blocks", "low_rank", "exact_dups"
    layers: int = 1


@dataclass(frozen=True)
class GateConfig:
    """One gate workload: n_c chunks of N float32 latents."""

    name: str
    n_chunks: int
    N: int
    T: int
    m: int
    eps: Tuple[float, ...]
    kind: str  # "gaussian" (v ~ N(0,1)*scale, dt=-1/T) or "toy" (flow-matching toy)
    p: float = 1.0
    x0_std: Tuple[float, ...] = field(default_factory=tuple)
    v_scale: Tuple[float, ...] = field(default_factory=tuple)
    stagger: int = 0  # chunk c starts at global step stagger*c
    latent_shape: Tuple[int, ...] = field(default_factory=tuple)


KV_CONFIGS = {
    # H=2, d=64, 256 queries, 1024 AR(1) keys (rho 0.9, innovation 0.436), fp32.
    "tiny_fp32": KVConfig("tiny_fp32", H=2, d=64, Lq=256, Lk=1024, B=256, lam=(0.5,),
                          pool=7, dtype="f32", rho=0.9, noise=0.436),
    # One bf16 layer: 4096 queries (one active chunk), 4 clean chunks of 4096 keys.
    "bf16_layer": KVConfig("bf16_layer", H=24, d=128, Lq=4096, Lk=16384, B=8192, lam=(0.5,),
                           pool=7, dtype="bf16", rho=0.95, structure="near_dup_blocks"),
    # 40 heads, 21x39x10 = 8190 queries, 4 clean chunks of 8190 keys.
    "bf16_large_head": KVConfig("bf16_large_head", H=40, d=128, Lq=8190, Lk=32760, B=16380,
                                lam=(0.3, 0.5, 0.7), pool=7, dtype="bf16", rho=0.9,
                                structure="low_rank"),
    # 16 clean chunks of 8192 keys, 25% exact duplicate K/V rows.
    "long_history": KVConfig("long_history", H=40, d=128, Lq=8192, Lk=131072, B=32768,
                             lam=(0.5,), pool=7, dtype="bf16", rho=0.97, structure="exact_dups"),
}
# Full-step sweep: 40 layers x H=40 at L_k in {4K, 16K, 64K, 128K}, B = L_k/4.
for _lk in (4096, 16384, 65536, 131072):
    KV_CONFIGS[f"sweep_lk{_lk}"] = KVConfig(
        f"sweep_lk{_lk}", H=40, d=128, Lq=4096, Lk=_lk, B=_lk // 4, lam=(0.5,), pool=7,
        dtype="bf16", rho=0.95, layers=40)

GATE_CONFIGS = {
    # 4 chunks of 1024x16 latents, v ~ N(0,1) * {0.5,1,2,4}, T=10, m=2, eps=0.05.
    "tiny_fp32": GateConfig("tiny_fp32", n_chunks=4, N=1024 * 16, T=10, m=2, eps=(0.05,),
                            kind="gaussian", v_scale=(0.5, 1.0, 2.0, 4.0),
                            latent_shape=(1024, 16)),
    # 4 chunks of 24x45x45x16 latents, T=30, m=5 (MAGI-1), eps=0.01 (MAGI-1 slow).
    "bf16_layer": GateConfig("bf16_layer", n_chunks=4, N=24 * 45 * 45 * 16, T=30, m=5,
                             eps=(0.01,), kind="toy", p=2.0, x0_std=(0.05, 0.1, 0.2, 0.4),
                             latent_shape=(24, 45, 45, 16)),
    # 8 chunks of 5x60x104x16 latents, T=30, m=4 (SkyReels-V2), eps 0.1 / 0.15.
    "bf16_large_head": GateConfig("bf16_large_head", n_chunks=8, N=5 * 60 * 104 * 16, T=30,
                                  m=4, eps=(0.1, 0.15), kind="toy", p=2.0,
                                  x0_std=(0.05, 0.1, 0.2, 0.4, 0.05, 0.1, 0.2, 0.4),
                                  latent_shape=(5, 60, 104, 16)),
    # 16 chunks of 24x45x45x16 latents, T=50, p=2, chunk c starts at global step 3c.
    "full_step_sweep": GateConfig("full_step_sweep", n_chunks=16, N=24 * 45 * 45 * 16, T=50,
                                  m=5, eps=(0.01,), kind="toy", p=2.0,
                                  x0_std=tuple(0.05 * (1 + (c % 4)) for c in range(16)),
                                  stagger=3, latent_shape=(24, 45, 45, 16)),
}


@dataclass(frozen=True)
class CacheConfig:
    """A stream of chunks entering the fixed KV buffer B_budget + C per head:
    C tokens per chunk, L_q queries of the chunk denoising at each commit."""

    name: str
    H: int
    d: int
    C: int
    B_budget: int
    n_chunks: int
    Lq: int
    lam: float
    pool: int
    dtype: str
    rho: float


CACHE_CONFIGS = {
    # 2 heads, d=64, chunks of 48 tokens, budget 2 chunks, 6 chunks, float32.
    "tiny_fp32_stream": CacheConfig("tiny_fp32_stream", H=2, d=64, C=48, B_budget=96,
                                    n_chunks=6, Lq=40, lam=0.5, pool=3, dtype="f32", rho=0.9),
    # 4 heads, d=128, chunks of 1024 tokens, budget 4 chunks, 8 chunks, bf16.
    "bf16_stream": CacheConfig("bf16_stream", H=4, d=128, C=1024, B_budget=4096, n_chunks=8,
                               Lq=256, lam=0.5, pool=7, dtype="bf16", rho=0.95),
    # Chunk sizes that do not divide the budget: the first compression scores
    # fewer than B_budget + C candidates.
    "tiny_fp32_ragged": CacheConfig("tiny_fp32_ragged", H=2, d=64, C=37, B_budget=100,
                                    n_chunks=7, Lq=40, lam=0.5, pool=3, dtype="f32", rho=0.9),
    "bf16_ragged": CacheConfig("bf16_ragged", H=3, d=128, C=300, B_budget=1000, n_chunks=6,
                               Lq=96, lam=0.5, pool=7, dtype="bf16", rho=0.95),
}


def _rng(seed, role, layer=0, head=0):
    return np.random.default_rng([int(seed), role, int(layer), int(head)])


def _ar1(rng, L, d, rho, noise):
    """AR(1) walk along tokens: x_0 ~ N(0,I), x_j = rho*x_{j-1} + noise*n_j.
    Returns a C-contiguous float64 [L, d] array."""
    n = rng.standard_normal((d, L), dtype=np.float32).astype(np.float64)
    n[:, 0] /= noise  # so that the filter's first output is n_0 itself
    y = scipy.signal.lfilter([noise], [1.0, -rho], n, axis=1)
    return torch.from_numpy(y).t().contiguous().numpy()


def _keys_one_head(cfg: KVConfig, seed, layer, head):
    rho = cfg.rho
    noise = cfg.noise if cfg.noise is not None else float(np.sqrt(1.0 - rho * rho))
    rng = _rng(seed, _ROLE_K, layer, head)
    k = _ar1(rng, cfg.Lk, cfg.d, rho, noise)
    dup_src = None
    if cfg.structure == "near_dup_blocks":
        # Each clean chunk (4 of them): the second half is groups of 8 consecutive
        # near-duplicates base + 0.01*n, base = the AR value at the group's start.
        chunk = cfg.Lk // 4
        r2 = _rng(seed, _ROLE_DUP, layer, head)
        for c in range(4):
            lo = c * chunk + chunk // 2
            hi = (c + 1) * chunk
            for g0 in range(lo, hi, 8):
                g1 = min(g0 + 8, hi)
                base = k[g0].copy()
                k[g0:g1] = base + 0.01 * r2.standard_normal((g1 - g0, cfg.d))
    elif cfg.structure == "low_rank":
        # k_j = 0.8*ar_j + 0.6*U_h z_j, U_h entries N(0,1/16), z an AR(0.9) walk in R^16.
        r2 = _rng(seed, _ROLE_LOWRANK, layer, head)
        U = r2.standard_normal((cfg.d, 16)) / 4.0
        z = _ar1(r2, cfg.Lk, 16, 0.9, float(np.sqrt(1.0 - 0.81)))
        k = 0.8 * k + 0.6 * (z @ U.T)
    elif cfg.structure == "exact_dups":
        # A seeded 25% of positions copy the K and V row of a uniformly chosen
        # non-duplicate position.
        r2 = _rng(seed, _ROLE_DUP, layer, head)
        n_dup = cfg.Lk // 4
        perm = r2.permutation(cfg.Lk)
        dups = np.sort(perm[:n_dup])
        originals = np.sort(perm[n_dup:])
        src = originals[r2.integers(0, originals.size, size=n_dup)]
        k[dups] = k[src]
        dup_src = (dups, src)
    return k.astype(np.float32), dup_src


def kv_head(cfg: KVConfig, seed=0, layer=0, head=0):
    """Q, K, V of one head as float32 numpy arrays ([L_q,d], [L_k,d], [L_k,d]),
    already rounded to bf16 when the workload is bf16."""
    k, dup_src = _keys_one_head(cfg, seed, layer, head)
    q = _rng(seed, _ROLE_Q, layer, head).standard_normal((cfg.Lq, cfg.d), dtype=np.float32)
    v = _rng(seed, _ROLE_V, layer, head).standard_normal((cfg.Lk, cfg.d), dtype=np.float32)
    if dup_src is not None:
        dups, src = dup_src
        v[dups] = v[src]
    if cfg.dtype == "bf16":
        q, k, v = (_round_bf16(a) for a in (q, k, v))
    return q, k, v


def _round_bf16(a):
    return torch.from_numpy(a).to(torch.bfloat16).float().numpy()


def kv_inputs(cfg: KVConfig, seed=0, layer=0, heads: Optional[Sequence[int]] = None):
    """Q [H,L_q,d], K [H,L_k,d], V [H,L_k,d] as torch CPU tensors in the
    workload's dtype (torch.bfloat16 or torch.float32).  ``heads`` selects a
    subset (default: all heads)."""
    heads = list(range(cfg.H)) if heads is None else list(heads)
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    Q = torch.empty(len(heads), cfg.Lq, cfg.d, dtype=tdt)
    K = torch.empty(len(heads), cfg.Lk, cfg.d, dtype=tdt)
    V = torch.empty(len(heads), cfg.Lk, cfg.d, dtype=tdt)

    def one(i):
        q, k, v = kv_head(cfg, seed, layer, heads[i])
        Q[i] = torch.from_numpy(q)
        K[i] = torch.from_numpy(k)
        V[i] = torch.from_numpy(v)

    # heads are independent streams: draw them on a few threads
    workers = max(1, min(len(heads), (os.cpu_count() or 2) // 2, 8))
    with ThreadPoolExecutor(workers) as ex:
        list(ex.map(one, range(len(heads))))
    return Q, K, V


# ---------------------------------------------------------------------------
# Gate inputs
# ---------------------------------------------------------------------------
def _sigma(t, T, p):
    return (t / T) ** p


def gate_initial(cfg: GateConfig, seed=0):
    """Initial latents X [n_c, N] float32 (pure noise for every chunk)."""
    x = np.empty((cfg.n_chunks, cfg.N), dtype=np.float32)
    for c in range(cfg.n_chunks):
        x[c] = _rng(seed, _ROLE_GATE_NOISE, 0, c).standard_normal(cfg.N, dtype=np.float32)
    return x


def gate_velocity(cfg: GateConfig, seed=0, draw=0):
    """Velocity v [n_c, N] float32.

    ``toy``: the exact flow-matching velocity x0 - noise of the single-point
    toy x_s = s*x0 + (1-s)*noise, with x0 ~ N(0, x0_std[c]^2) (constant along
    the trajectory).  ``gaussian``: a fresh N(0,1)*v_scale[c] draw per ``draw``
    index (a recompute produces a new draw; a reuse re-applies the old one)."""
    v = np.empty((cfg.n_chunks, cfg.N), dtype=np.float32)
    for c in range(cfg.n_chunks):
        if cfg.kind == "toy":
            x0 = _rng(seed, _ROLE_GATE_X0, 0, c).standard_normal(cfg.N) * cfg.x0_std[c]
            eps = _rng(seed, _ROLE_GATE_NOISE, 0, c).standard_normal(cfg.N, dtype=np.float32)
            v[c] = (x0 - eps.astype(np.float64)).astype(np.float32)
        else:
            g = _rng(seed, _ROLE_GATE_V, draw, c).standard_normal(cfg.N, dtype=np.float32)
            v[c] = g * np.float32(cfg.v_scale[c])
    return v


def gate_step_counters(cfg: GateConfig, global_step):
    """Per-chunk step counters at a global step: step_c = g - stagger*c, or -1
    when the chunk has not started or has finished its T steps."""
    s = np.array([global_step - cfg.stagger * c for c in range(cfg.n_chunks)], dtype=np.int32)
    s[(s < 0) | (s >= cfg.T)] = -1
    return s


def gate_dt(cfg: GateConfig, steps):
    """Per-chunk signed step dt [n_c] float32 for the given step counters.

    ``toy``: sigma(s+1) - sigma(s) with sigma(t) = (t/T)^p (noise at t=0, data
    at t=T).  ``gaussian``: -1/T.  Inactive chunks get 0."""
    dt = np.zeros(cfg.n_chunks, dtype=np.float32)
    for c, s in enumerate(steps):
        if s < 0:
            continue
        if cfg.kind == "toy":
            dt[c] = _sigma(s + 1, cfg.T, cfg.p) - _sigma(s, cfg.T, cfg.p)
        else:
            dt[c] = -1.0 / cfg.T
    return dt


def cache_inputs(cfg: CacheConfig, seed=0):
    """Chunk K and V ([n_chunks] of [H, C, d]) and, per chunk, the queries of
    the chunk denoising when it finishes ([n_chunks] of [H, L_q, d]), torch
    CPU tensors.  The keys are one AR(1) walk across the whole stream, cut into
    chunks, so consecutive chunks are correlated as video tokens are."""
    kv = KVConfig(cfg.name, H=cfg.H, d=cfg.d, Lq=cfg.Lq * cfg.n_chunks, Lk=cfg.C * cfg.n_chunks,
                  B=cfg.B_budget, lam=(cfg.lam,), pool=cfg.pool, dtype=cfg.dtype, rho=cfg.rho)
    Q, K, V = kv_inputs(kv, seed=seed)
    C, Lq = cfg.C, cfg.Lq
    ks = [K[:, i * C:(i + 1) * C].contiguous() for i in range(cfg.n_chunks)]
    vs = [V[:, i * C:(i + 1) * C].contiguous() for i in range(cfg.n_chunks)]
    qs = [Q[:, i * Lq:(i + 1) * Lq].contiguous() for i in range(cfg.n_chunks)]
    return ks, vs, qs

