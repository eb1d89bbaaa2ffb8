"""Helpers for comparing the CUDA path with the CPU oracle.

Tolerances (relative L2 over the compared tensor):
  float32 path:  O, LSE, dQ, dK, dV <= 1e-5
  bf16 path:     O, LSE <= 2e-3;  dQ, dK, dV <= 1e-2;  decode o <= 2e-3
Keep decisions must match exactly, except tiles whose contribution ratio is
within 1e-3 relative of the threshold (|margin| <= ln(1 + 1e-3)) and, in the
forward, the later tiles of the same query block after such a flip (their
state differs). Such flips are counted and reported. Both decisions are
correct there, so only what the flip does not touch is compared:
  forward flip in query block i   -> O, LSE rows of block i; dQ rows of block
                                     i; dK, dV rows of every key block that
                                     block i keeps in the backward (either
                                     side), since their sums include rows of i;
  backward flip of tile (i, j)    -> dQ rows of block i, dK, dV rows of block j.
Every other row is compared, and the callers assert how many were.
"""

from __future__ import annotations

import math

import numpy as np

NEAR = math.log1p(1e-3)
TOL = {"f32": {"O": 1e-5, "LSE": 1e-5, "grad": 1e-5},
       "bf16": {"O": 2e-3, "LSE": 2e-3, "grad": 1e-2, "decode": 2e-3}}


def rel_l2(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def compare_fwd_keep(gpu_keep, ref_keep, ref_margin, row_offset=0):
    """Forward keep sets of one slice: rows are query blocks row_offset,
    row_offset + 1, ...; columns are key blocks. Returns (n_near, bad_rows)
    where bad_rows are local row indices with an allowed flip. Raises
    AssertionError on a disallowed mismatch."""
    n_near = 0
    bad_blocks = []
    for li in range(ref_keep.shape[0]):
        i = li + row_offset
        flipped = False
        for j in range(i, -1, -1):
            g, r = int(gpu_keep[li, j]), int(ref_keep[li, j])
            if g == r:
                continue
            if flipped:
                continue  # downstream of an allowed flip in this block
            mu = ref_margin[li, j]
            assert abs(mu) <= NEAR, f"keep mismatch at ({i},{j}) margin {mu}"
            n_near += 1
            flipped = True
        if flipped:
            bad_blocks.append(li)
    return n_near, bad_blocks


def compare_bwd_keep(gpu_keep, ref_keep, ref_margin, skip_blocks=()):
    """Backward keep sets of one slice (rows = query blocks, columns = key
    blocks). Rows in ``skip_blocks`` (forward flips: their LSE differs) are
    not compared. Returns the list of allowed near-threshold flips (i, j);
    raises AssertionError on any other mismatch."""
    nb = ref_keep.shape[0]
    flips = []
    tril = np.tril(np.ones((nb, nb), bool))
    diff = (gpu_keep.astype(bool) != ref_keep.astype(bool)) & tril
    for i, j in zip(*np.nonzero(diff)):
        if i in skip_blocks:
            continue
        assert abs(ref_margin[i, j]) <= NEAR, f"bwd keep mismatch at ({i},{j}) margin {ref_margin[i, j]}"
        flips.append((int(i), int(j)))
    return flips


def grad_row_masks(L, tile, fwd_bad, bwd_flips, gpu_bkeep, ref_bkeep):
    """Rows of dQ (query rows) and of dK, dV (key rows) that no allowed flip
    touches (see the module docstring)."""
    qmask = np.ones(L, bool)
    kmask = np.ones(L, bool)
    either = gpu_bkeep.astype(bool) | ref_bkeep.astype(bool)
    for i in fwd_bad:
        qmask[i * tile:(i + 1) * tile] = False
        for j in np.nonzero(either[i, :i + 1])[0]:
            kmask[j * tile:(j + 1) * tile] = False
    for i, j in bwd_flips:
        qmask[i * tile:(i + 1) * tile] = False
        kmask[j * tile:(j + 1) * tile] = False
    return qmask, kmask


class Coverage:
    """What a test compared: rows per tensor (compared, total) and the
    near-threshold flips it allowed. ``report()`` prints one line (visible
    with pytest -s or in the failure output); ``require()`` asserts that at
    least ``frac`` of the rows of every tensor were compared."""

    def __init__(self, name):
        self.name = name
        self.rows = {}
        self.flips = {"fwd": 0, "bwd": 0, "decode": 0}
        self.slices = 0

    def add(self, tensor, mask):
        c, t = self.rows.get(tensor, (0, 0))
        self.rows[tensor] = (c + int(np.count_nonzero(mask)), t + int(np.size(mask)))

    def report(self):
        parts = [f"{k} {c}/{t}" for k, (c, t) in sorted(self.rows.items())]
        print(f"[coverage] {self.name}: slices {self.slices}; rows compared " + ", ".join(parts) +
              f"; near-threshold flips fwd {self.flips['fwd']} bwd {self.flips['bwd']} "
              f"decode {self.flips['decode']}", flush=True)

    def require(self, frac):
        self.report()
        assert self.rows, "nothing compared"
        for k, (c, t) in self.rows.items():
            assert c >= frac * t, f"{self.name}: only {c} of {t} rows of {k} compared"


def row_mask(L, tile, bad_blocks):
    m = np.ones(L, bool)
    for i in bad_blocks:
        m[i * tile:(i + 1) * tile] = False
    return m


def as_f64(t):
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def compare_decode_keep(gpu_keep, ref_keep, ref_margin):
    """Decode keep sequence of one group: tiles visited newest first. Returns
    True if an allowed near-threshold flip happened (later tiles unchecked;
    the group's output then differs legitimately: its heads share the
    decisions)."""
    nt = len(ref_keep)
    for t in range(nt - 1, -1, -1):
        if int(gpu_keep[t]) == int(ref_keep[t]):
            continue
        assert abs(ref_margin[t]) <= NEAR, f"decode keep mismatch at tile {t} margin {ref_margin[t]}"
        return True
    return False
