"""Retained slots per query: the pages' "post-score key slots per query"
(jaehun.me review, "2) One tolerance holds across contexts"), read as the
mean over query rows of the legal keys (key <= query) that lie in kept tiles.

Every slots-per-query figure and the retained term of every effective
TFLOP/s figure in bench.py comes from ``bench.retained_pairs``; it is pinned
here to ``oracle.retained_slots``, and that to a pure-Python enumeration of
(row, key) pairs. CPU only.
"""

from __future__ import annotations

import numpy as np
import pytest

import oracle

torch = pytest.importorskip("torch")

import bench  # noqa: E402


def enumerate_slots(keep, L, tile):
    """Mean over rows r < L of #{keys c <= r : tile (r // tile, c // tile) kept}."""
    total = 0
    for r in range(L):
        for c in range(r + 1):
            if keep[r // tile, c // tile]:
                total += 1
    return total / L


def random_keep(rng, nb, p):
    keep = (rng.random((nb, nb)) < p).astype(np.uint8)
    return np.tril(keep)


def pack_rows(keep):
    """(..., nb, nb) 0/1 -> (..., nb, ceil(nb/32)) int32 words, bit j % 32 of
    word j // 32 = column j (the library's keep-bit layout)."""
    nb = keep.shape[-1]
    nw = (nb + 31) // 32
    words = np.zeros(keep.shape[:-1] + (nw,), dtype=np.uint32)
    for j in range(nb):
        words[..., j // 32] |= keep[..., j].astype(np.uint32) << np.uint32(j % 32)
    return torch.from_numpy(words.view(np.int32))


@pytest.mark.parametrize("L,tile", [(1, 1), (7, 1), (10, 3), (11, 3), (128, 128), (130, 128),
                                    (300, 128), (383, 128), (40, 7)])
def test_oracle_retained_slots_is_the_enumeration(L, tile):
    rng = np.random.default_rng(L * 31 + tile)
    nb = oracle.n_blocks(L, tile)
    for p in (0.0, 0.3, 1.0):
        keep = random_keep(rng, nb, p)
        assert oracle.retained_slots(keep, L, tile) == pytest.approx(enumerate_slots(keep, L, tile),
                                                                     abs=0, rel=1e-15)


def test_retained_slots_closed_forms():
    # every tile kept: all L(L+1)/2 legal pairs
    for L, tile in ((1000, 128), (1024, 128), (129, 128), (13, 4)):
        nb = oracle.n_blocks(L, tile)
        full = np.tril(np.ones((nb, nb), np.uint8))
        assert oracle.retained_slots(full, L, tile) * L == L * (L + 1) // 2
        # only the diagonal tiles: sum over blocks of r(r+1)/2 rows-by-keys
        diag = np.eye(nb, dtype=np.uint8)
        rows = [min(L - i * tile, tile) for i in range(nb)]
        assert oracle.retained_slots(diag, L, tile) * L == sum(r * (r + 1) // 2 for r in rows)


@pytest.mark.parametrize("L", [128, 1000, 1536, 2049, 4096 + 17])
def test_bench_retained_pairs_equals_oracle(L):
    """bench.retained_pairs over a [B, H, nb, nw] bit stack (B=2, H=3, random
    keep sets with a ragged last block) equals L times the oracle's slots per
    query summed over slices."""
    tile = 128
    nb = oracle.n_blocks(L, tile)
    rng = np.random.default_rng(L)
    keeps = np.stack([np.stack([random_keep(rng, nb, p) for p in (0.05, 0.5, 1.0)])
                      for _ in range(2)])  # (2, 3, nb, nb)
    for b in range(2):
        for h in range(3):
            keeps[b, h][np.arange(nb), np.arange(nb)] = 1  # the forward keeps its diagonal
    bits = pack_rows(keeps)
    got = bench.retained_pairs(bits, L, tile)
    want = sum(oracle.retained_slots(keeps[b, h], L, tile) * L for b in range(2) for h in range(3))
    assert got == round(want)
