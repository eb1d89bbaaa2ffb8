"""Seeded synthetic inputs for the MALA workloads.

This module is shared by the CPU oracle tests and the CUDA path. It holds only
the input recipe (random numbers and their arrangement); none of the attention
arithmetic lives here.

Recipe (the pages' inputs were model activations, which are not available; this
stands in for them, with the structure the pages attribute to long-context
attention: mass concentrated on local keys, a sink token and a few retrieval
positions -- MassAlloc Attention, jaehun.me review, "Background" and section 3
"One tolerance holds across contexts"):

* one independent stream per (config, sequence): numpy ``default_rng(seed)``
  with ``seed = config_seed * 1000 + sequence_index`` where
  ``sequence_index = b * H + h``;
* latent AR(1): ``x_0 = e_0``, ``x_t = rho x_{t-1} + sqrt(1 - rho^2) e_t``,
  ``e_t ~ N(0, I_d)`` drawn as one ``(d, L)`` block (column t is ``e_t``);
* ``Q = K = 2.5 x``; a sink: ``K_0 += 6 u`` and ``Q_t += 1.5 u`` for all t,
  ``u`` a unit vector drawn once per config from seed ``config_seed*1000+999``;
* retrieval pairs: ``n_pairs`` distinct queries ``i`` in ``[258, L)`` (sorted)
  and, for each, a fresh key position ``j`` in ``[1, i - 256)`` (no ``j``
  reused); ``K_j = 2.5 * sqrt(d) * Q_i / |Q_i|`` using the post-sink ``Q_i``;
* ``V ~ N(0, 1)`` then ``dO ~ N(0, 1)``, both ``(L, d)``, drawn after the pairs.

Everything is produced in float64 and cast by the caller.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
from scipy.signal import lfilter

__all__ = [
    "PrefillConfig",
    "DecodeConfig",
    "CONFIGS",
    "unit_vector",
    "prefill_sequence",
    "prefill_inputs",
    "decode_group",
    "decode_inputs",
]


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    config_seed: int
    B: int
    H: int
    L: int
    d: int
    tile: int
    dtype: str  # "f32" or "bf16"
    rho: float
    n_pairs: int
    taus: tuple = (1.0,)


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    config_seed: int
    B: int
    Hq: int
    Hkv: int
    Lc: int
    d: int
    tile: int
    rho: float
    n_pairs: int          # retrieval pairs planted by the sequence generator
    n_query_targets: int  # cache positions per query head aimed at that head
    taus: tuple = (1.0,)


def _cfg2(L: int) -> PrefillConfig:
    return PrefillConfig(f"sweep_L{L}", 2, 1, 16, L, 128, 128, "bf16", 0.97,
                         L // 128, (1.0, 0.0))


CONFIGS = {
    "tiny_f32": PrefillConfig("tiny_f32", 0, 1, 1, 1024, 64, 64, "f32", 0.97, 8,
                              (1.0, 0.0)),
    "matched_8k": PrefillConfig("matched_8k", 1, 1, 8, 8192, 128, 128, "bf16",
                                0.97, 64, (1.0,)),
    **{f"sweep_L{L}": _cfg2(L) for L in (1024, 2048, 4096, 8192, 16384, 32768)},
    "long_128k": PrefillConfig("long_128k", 3, 1, 8, 131072, 128, 128, "bf16",
                               0.98, 1024, (1.0, 0.0)),
    "decode_128k": DecodeConfig("decode_128k", 4, 16, 32, 8, 131072, 128, 128,
                                0.98, 1024, 4, (1.0,)),
}


def unit_vector(config_seed: int, d: int) -> np.ndarray:
    """The per-config sink direction u (unit norm, float64)."""
    rng = np.random.default_rng(config_seed * 1000 + 999)
    u = rng.standard_normal(d)
    return u / np.linalg.norm(u)


def _latent(rng: np.random.Generator, L: int, d: int, rho: float) -> np.ndarray:
    """AR(1) latent x of shape (L, d), float64."""
    e = rng.standard_normal((d, L))
    c = math.sqrt(1.0 - rho * rho)
    w = e * c
    w[:, 0] = e[:, 0]  # x_0 = e_0 (stationary start)
    x = lfilter([1.0], [1.0, -rho], w, axis=1)
    return np.ascontiguousarray(x.T)


def _plant_pairs(rng, Q, K, n_pairs, L, d):
    """Retrieval pairs: K_j <- 2.5 sqrt(d) Q_i/|Q_i| for chosen (i, j)."""
    lo = 258
    if n_pairs <= 0 or L <= lo:
        return np.zeros((0, 2), dtype=np.int64)
    n_pairs = min(n_pairs, L - lo)
    qs = np.sort(rng.choice(np.arange(lo, L), size=n_pairs, replace=False))
    used = set()
    pairs = []
    for i in qs:
        hi = int(i) - 256  # j in [1, hi)
        j = None
        for _ in range(64):
            cand = int(rng.integers(1, hi))
            if cand not in used:
                j = cand
                break
        if j is None:  # dense corner: take the smallest free position
            free = [c for c in range(1, hi) if c not in used]
            if not free:
                continue
            j = free[0]
        used.add(j)
        qi = Q[i]
        K[j] = 2.5 * math.sqrt(d) * qi / np.linalg.norm(qi)
        pairs.append((int(i), j))
    return np.asarray(pairs, dtype=np.int64).reshape(-1, 2)


def prefill_sequence(config_seed: int, seq_index: int, L: int, d: int,
                     rho: float, n_pairs: int, u: np.ndarray | None = None,
                     with_grad: bool = True):
    """One (b, h) slice: returns dict of float64 (L, d) arrays Q, K, V, dO
    (dO only when ``with_grad``) and the planted ``pairs`` (n, 2)."""
    if u is None:
        u = unit_vector(config_seed, d)
    rng = np.random.default_rng(config_seed * 1000 + seq_index)
    x = _latent(rng, L, d, rho)
    Q = 2.5 * x
    K = Q.copy()
    K[0] += 6.0 * u
    Q += 1.5 * u
    pairs = _plant_pairs(rng, Q, K, n_pairs, L, d)
    V = rng.standard_normal((L, d))
    out = {"Q": Q, "K": K, "V": V, "pairs": pairs}
    if with_grad:
        out["dO"] = rng.standard_normal((L, d))
    return out


def prefill_inputs(cfg: PrefillConfig, L: int | None = None,
                   heads: list | None = None, with_grad: bool = True):
    """Stacked float64 arrays of shape (B, H, L, d) for a prefill config.

    ``L`` overrides the config's length (the same streams, shorter prefix is
    *not* implied: a different L is a different draw). ``heads`` restricts
    generation to the listed flat (b*H+h) indices (others are zero)."""
    L = cfg.L if L is None else L
    u = unit_vector(cfg.config_seed, cfg.d)
    names = ["Q", "K", "V"] + (["dO"] if with_grad else [])
    out = {n: np.zeros((cfg.B, cfg.H, L, cfg.d)) for n in names}
    n_seq = cfg.B * cfg.H
    for s in range(n_seq) if heads is None else heads:
        b, h = divmod(s, cfg.H)
        seq = prefill_sequence(cfg.config_seed, s, L, cfg.d, cfg.rho,
                               cfg.n_pairs, u, with_grad)
        for n in names:
            out[n][b, h] = seq[n]
    return out


def decode_group(cfg: DecodeConfig, b: int, g: int, u: np.ndarray | None = None):
    """KV cache of one (b, kv-head g) and the G = Hq/Hkv query vectors of its
    group. Returns dict K, V (Lc, d) float64, q (G, d) float64, targets (G, n).

    The cache is the prefill recipe with ``L = Lc`` (its Q discarded). Each
    group query is ``q = 2.5 (rho x_{Lc-1} + sqrt(1-rho^2) e) + 1.5 u`` with a
    fresh ``e``; ``n_query_targets`` fresh cache positions ``j < Lc - 256``
    per query head are set to ``2.5 sqrt(d) q/|q|``."""
    if u is None:
        u = unit_vector(cfg.config_seed, cfg.d)
    G = cfg.Hq // cfg.Hkv
    Lc, d, rho = cfg.Lc, cfg.d, cfg.rho
    seq_index = b * cfg.Hkv + g
    rng = np.random.default_rng(cfg.config_seed * 1000 + seq_index)
    x = _latent(rng, Lc, d, rho)
    Q = 2.5 * x
    K = Q.copy()
    K[0] += 6.0 * u
    Q += 1.5 * u
    pairs = _plant_pairs(rng, Q, K, cfg.n_pairs, Lc, d)
    V = rng.standard_normal((Lc, d))
    c = math.sqrt(1.0 - rho * rho)
    q = 2.5 * (rho * x[Lc - 1][None, :] + c * rng.standard_normal((G, d))) + 1.5 * u
    used = set(int(j) for j in pairs[:, 1]) if len(pairs) else set()
    targets = np.zeros((G, cfg.n_query_targets), dtype=np.int64)
    hi = max(2, Lc - 256)
    for h in range(G):
        for t in range(cfg.n_query_targets):
            for _ in range(1000):
                j = int(rng.integers(1, hi))
                if j not in used:
                    break
            used.add(j)
            K[j] = 2.5 * math.sqrt(d) * q[h] / np.linalg.norm(q[h])
            targets[h, t] = j
    return {"K": K, "V": V, "q": q, "targets": targets}


def decode_inputs(cfg: DecodeConfig, groups: list | None = None):
    """Stacked float64 arrays q (B, Hq, d), K and V (B, Hkv, Lc, d).
    ``groups`` restricts generation to the listed flat (b*Hkv+g) indices."""
    G = cfg.Hq // cfg.Hkv
    u = unit_vector(cfg.config_seed, cfg.d)
    q = np.zeros((cfg.B, cfg.Hq, cfg.d))
    K = np.zeros((cfg.B, cfg.Hkv, cfg.Lc, cfg.d))
    V = np.zeros_like(K)
    for s in range(cfg.B * cfg.Hkv) if groups is None else groups:
        b, g = divmod(s, cfg.Hkv)
        grp = decode_group(cfg, b, g, u)
        K[b, g], V[b, g] = grp["K"], grp["V"]
        q[b, g * G:(g + 1) * G] = grp["q"]
    return {"q": q, "K": K, "V": V}
