"""CPU oracle for MALA (MassAlloc Attention) -- test infrastructure only.

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package. The product path (the CUDA library and its binding)
never imports it, and it imports nothing from the product.

The arithmetic lives in ``mala_oracle.c`` (float64, scalar loops, OpenMP over
independent query/key blocks). This module compiles it with gcc on first use
and wraps it with numpy-facing helpers over (B, H, L, d) stacks.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mala_oracle.c")
_LIB = os.path.join(_HERE, "libmala_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_ip = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile the oracle shared library (gcc, OpenMP). Returns its path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # MALA_ORACLE_LIB lets the mutation tests load a deliberately
            # broken copy of the oracle and check that the pins catch it.
            alt = os.environ.get("MALA_ORACLE_LIB")
            lib = ctypes.CDLL(alt if alt else build())
            c_int, c_double = ctypes.c_int, ctypes.c_double
            lib.mala_oracle_threads.argtypes = [c_int]
            lib.mala_oracle_threads.restype = c_int
            lib.mala_oracle_fwd.argtypes = [_dp, _dp, _dp, c_int, c_int, c_int, c_double,
                                            c_double, c_int, _dp, _dp, _u8p, _dp, c_int, c_int]
            lib.mala_oracle_bwd.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, c_int, c_int, c_int,
                                            c_double, c_double, c_int, _ip, c_int, _ip, c_int,
                                            _dp, _dp, _dp, _u8p, _dp]
            lib.mala_oracle_decode.argtypes = [_dp, _dp, _dp, c_int, c_int, c_int, c_int, c_int,
                                               c_double, c_double, c_int, _dp, _u8p, _dp]
            lib.mala_oracle_dense_fwd.argtypes = [_dp, _dp, _dp, c_int, c_int, c_double, _dp, _dp]
            lib.mala_oracle_fwd_chunk.argtypes = [_dp, _dp, _dp, c_int, c_int, c_int, c_int,
                                                  c_double, c_double, _dp, _dp, _u8p, _dp]
            lib.mala_oracle_dense_bwd.argtypes = [_dp, _dp, _dp, _dp, c_int, c_int, c_double,
                                                  _dp, _dp, _dp]
            lib.mala_oracle_omitted_mass.argtypes = [_dp, _dp, c_int, c_int, c_int, c_double,
                                                     _u8p, _dp, _dp]
            for f in ("fwd", "bwd", "decode", "dense_fwd", "dense_bwd", "omitted_mass"):
                getattr(lib, "mala_oracle_" + f).restype = c_int
            _lib = lib
    return _lib


def threads(n: int = 0) -> int:
    """Set (n > 0) and return the OpenMP thread count the oracle uses."""
    return _load().mala_oracle_threads(int(n))


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a, t=_dp):
    return None if a is None else a.ctypes.data_as(t)


def n_blocks(L: int, T: int) -> int:
    return (L + T - 1) // T


def fwd(Q, K, V, tile, tau=1.0, scale=None, force_first=True, qblocks=None,
        want_margin=False):
    """MALA forward of one (L, d) slice.

    Returns dict O (L, d), LSE (L,), keep (nb, nb) uint8 (query block, key
    block), margin (nb, nb) if requested. ``qblocks=(lo, hi)`` restricts the
    work to query blocks [lo, hi); rows outside stay NaN and keep rows 0."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    L, d = Q.shape
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    nb = n_blocks(L, tile)
    lo, hi = (0, nb) if qblocks is None else qblocks
    O = np.full((L, d), np.nan)
    LSE = np.full(L, np.nan)
    keep = np.zeros((nb, nb), np.uint8)
    margin = np.full((nb, nb), np.nan) if want_margin else None
    _load().mala_oracle_fwd(_p(Q), _p(K), _p(V), L, d, tile, scale, float(tau),
                            int(force_first), _p(O), _p(LSE), _p(keep, _u8p),
                            _p(margin), int(lo), int(hi))
    out = {"O": O, "LSE": LSE, "keep": keep}
    if want_margin:
        out["margin"] = margin
    return out


def fwd_chunk(Q, K, V, tile, tau=1.0, scale=None, want_margin=False):
    """MALA forward of a prefill chunk appended to a KV cache: Q (Lq, d) are
    the last Lq positions of a sequence whose keys/values K, V are (Lk, d).
    Query row r sits at position Lk - Lq + r. Key tiles are aligned to the
    chunk's query blocks (tile k starts at position off + tile (k - koff),
    koff = ceil(off / tile)); keep / margin are (nbq, nbq + koff)."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    Lq, d = Q.shape
    Lk = K.shape[0]
    assert Lk >= Lq
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    nbq = n_blocks(Lq, tile)
    koff = n_blocks(Lk - Lq, tile)
    O = np.full((Lq, d), np.nan)
    LSE = np.full(Lq, np.nan)
    keep = np.zeros((nbq, nbq + koff), np.uint8)
    margin = np.full((nbq, nbq + koff), np.nan) if want_margin else None
    _load().mala_oracle_fwd_chunk(_p(Q), _p(K), _p(V), Lq, Lk, d, tile, scale, float(tau),
                                  _p(O), _p(LSE), _p(keep, _u8p), _p(margin))
    out = {"O": O, "LSE": LSE, "keep": keep, "koff": koff}
    if want_margin:
        out["margin"] = margin
    return out


def bwd(Q, K, V, O, dO, LSE, tile, tau=1.0, scale=None, force_first=False,
        qblocks=None, kblocks=None, want_margin=False):
    """MALA backward of one slice. ``qblocks``/``kblocks`` are lists of block
    indices for dQ and dK/dV (default: all). Rows not covered stay zero."""
    Q, K, V, O, dO, LSE = map(_f64, (Q, K, V, O, dO, LSE))
    L, d = Q.shape
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    nb = n_blocks(L, tile)
    qb = np.ascontiguousarray(np.arange(nb) if qblocks is None else qblocks, dtype=np.int32)
    kb = np.ascontiguousarray(np.arange(nb) if kblocks is None else kblocks, dtype=np.int32)
    dQ, dK, dV = np.zeros((L, d)), np.zeros((L, d)), np.zeros((L, d))
    keep = np.zeros((nb, nb), np.uint8)
    margin = np.full((nb, nb), np.nan) if want_margin else None
    _load().mala_oracle_bwd(_p(Q), _p(K), _p(V), _p(O), _p(dO), _p(LSE), L, d, tile, scale,
                            float(tau), int(force_first), _p(qb, _ip), len(qb), _p(kb, _ip),
                            len(kb), _p(dQ), _p(dK), _p(dV), _p(keep, _u8p), _p(margin))
    out = {"dQ": dQ, "dK": dK, "dV": dV, "keep": keep}
    if want_margin:
        out["margin"] = margin
    return out


def decode(q, Kc, Vc, tau=1.0, tile=128, scale=None, per_head=False,
           want_margin=False):
    """MALA decode step of one batch entry: q (Hq, d), Kc/Vc (Hkv, Lc, d).
    Returns o (Hq, d), keep (units, nt) and optionally margin."""
    q, Kc, Vc = _f64(q), _f64(Kc), _f64(Vc)
    Hq, d = q.shape
    Hkv, Lc, _ = Kc.shape
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    nt = n_blocks(Lc, tile)
    units = Hq if per_head else Hkv
    o = np.zeros((Hq, d))
    keep = np.zeros((units, nt), np.uint8)
    margin = np.full((units, nt), np.nan) if want_margin else None
    _load().mala_oracle_decode(_p(q), _p(Kc), _p(Vc), Hq, Hkv, Lc, d, tile, scale,
                               float(tau), int(per_head), _p(o), _p(keep, _u8p), _p(margin))
    out = {"o": o, "keep": keep}
    if want_margin:
        out["margin"] = margin
    return out


def dense_fwd(Q, K, V, scale=None):
    """Textbook causal softmax attention of one slice: O (L, d), LSE (L,)."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    L, d = Q.shape
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    O, LSE = np.zeros((L, d)), np.zeros(L)
    _load().mala_oracle_dense_fwd(_p(Q), _p(K), _p(V), L, d, scale, _p(O), _p(LSE))
    return {"O": O, "LSE": LSE}


def dense_bwd(Q, K, V, dO, scale=None):
    """Analytic gradients of textbook causal softmax attention of one slice."""
    Q, K, V, dO = map(_f64, (Q, K, V, dO))
    L, d = Q.shape
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    dQ, dK, dV = np.zeros((L, d)), np.zeros((L, d)), np.zeros((L, d))
    _load().mala_oracle_dense_bwd(_p(Q), _p(K), _p(V), _p(dO), L, d, scale, _p(dQ), _p(dK), _p(dV))
    return {"dQ": dQ, "dK": dK, "dV": dV}


def omitted_mass(Q, K, keep, LSE_dense, tile, scale=None):
    """Per-row dense probability mass that falls in skipped tiles."""
    Q, K, LSE_dense = _f64(Q), _f64(K), _f64(LSE_dense)
    L, d = Q.shape
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    mass = np.zeros(L)
    _load().mala_oracle_omitted_mass(_p(Q), _p(K), L, d, tile, scale, _p(keep, _u8p),
                                     _p(LSE_dense), _p(mass))
    return mass


def tile_row_max(Q, K, tile, qblocks=None):
    """Raw (unscaled) score maximum of every query row over every legal key
    tile: for query block i, key block j <= i and row r of block i,
        out[i][j, r] = max over key c of block j with c <= i*tile + r of Q[i*tile + r] . K[c].
    This is the quantity the backward's offline test compares with the final
    log-normalizer (MassAlloc Attention; jaehun.me review, "Backward: offline
    sparse probabilities": a tile stays iff some row's largest score clears
    LSE + ln tau - ln(position)). Rows past L are -inf.

    Returns {i: array (i + 1, tile)} for the query blocks in ``qblocks``
    (a (lo, hi) range; default all)."""
    Q, K = _f64(Q), _f64(K)
    L, d = Q.shape
    nb = n_blocks(L, tile)
    lo, hi = (0, nb) if qblocks is None else qblocks
    out = {}
    for i in range(lo, hi):
        r0, r1 = i * tile, min(L, (i + 1) * tile)
        S = Q[r0:r1] @ K[:r1].T                       # (rows, keys <= last row)
        rows = np.arange(r0, r1)[:, None]
        S[np.arange(r1)[None, :] > rows] = -np.inf    # causal mask
        m = np.full((i + 1, tile), -np.inf)
        for j in range(i + 1):
            c0, c1 = j * tile, min(r1, (j + 1) * tile)
            m[j, :r1 - r0] = S[:, c0:c1].max(axis=1)
        out[i] = m
    return out


def retained_slots(keep, L, tile):
    """Mean over query rows of the number of legal keys inside kept tiles
    (the pages' "post-score key slots per query")."""
    nb = n_blocks(L, tile)
    total = 0
    for i in range(nb):
        r0, r1 = i * tile, min(L, (i + 1) * tile)
        for j in range(i + 1):
            if not keep[i, j]:
                continue
            c0, c1 = j * tile, min(L, (j + 1) * tile)
            if j < i:
                total += (r1 - r0) * (c1 - c0)
            else:  # diagonal: row r sees keys c0..r
                total += sum(r - c0 + 1 for r in range(r0, r1))
    return total / L
