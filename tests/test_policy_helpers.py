"""The host analysis behind bench.py's matched-work study (CPU only): its
per-tile dense mass agrees with the oracle's omitted mass, and its
restricted output with the oracle's own forward on the oracle's keep set
(MassAlloc Attention; jaehun.me review, "Matched-work study")."""

from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth

pytest.importorskip("torch")

import bench  # noqa: E402

T = 128


@pytest.fixture(scope="module")
def slice_1k():
    cfg = synth.CONFIGS["matched_8k"]
    x = synth.prefill_inputs(cfg, L=1100, heads=[2], with_grad=False)
    return {n: bench.bf16_round(x[n][0, 2]) for n in ("Q", "K", "V")}


def test_row_tile_mass_is_a_distribution(slice_1k):
    Q, K = slice_1k["Q"], slice_1k["K"]
    P, rm = bench.dense_row_tile_mass(Q, K, T, 1 / np.sqrt(128))
    L = Q.shape[0]
    np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-12)
    np.testing.assert_allclose(rm.sum(axis=1), 1.0, atol=1e-12)
    assert np.all(np.triu(P, 1) == 0)
    # a row puts no mass on key tiles after its own block
    blk = np.arange(L) // T
    assert np.all(rm[np.arange(rm.shape[1])[None, :] > blk[:, None]] == 0)
    bm = bench.block_mass(rm, T)
    np.testing.assert_allclose(bm.sum(axis=1), [min(T, L - i * T) for i in range(bm.shape[0])],
                               atol=1e-9)


def test_mass_and_output_match_the_oracle(slice_1k):
    Q, K, V = slice_1k["Q"], slice_1k["K"], slice_1k["V"]
    f = oracle.fwd(Q, K, V, tile=T, tau=1.0)
    dense = oracle.dense_fwd(Q, K, V)
    om_ref = oracle.omitted_mass(Q, K, f["keep"], dense["LSE"], T)
    P, rm = bench.dense_row_tile_mass(Q, K, T, 1 / np.sqrt(128))
    O, om = bench.restricted_output(P, V, f["keep"], T)
    np.testing.assert_allclose(om, om_ref, rtol=0, atol=1e-12)
    # the rule's output is the softmax restricted to its keep set
    np.testing.assert_allclose(O, f["O"], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(P @ V, dense["O"], rtol=1e-9, atol=1e-12)


def test_policies_spend_the_same_budget():
    rng = np.random.default_rng(3)
    nb = 12
    counts = np.array([min(i + 1, int(rng.integers(1, 5))) for i in range(nb)])
    score = rng.random((nb, nb))
    for keep in (bench.position_static_keep(counts), bench.top_keep(score, counts)):
        assert np.array_equal(keep.sum(axis=1), counts)
        assert np.all(np.triu(keep, 1) == 0)
    st = bench.position_static_keep(counts)
    assert all(st[i, i] == 1 for i in range(nb))
    assert all(st[i, 0] == 1 for i in range(1, nb) if counts[i] >= 2)
    top = bench.top_keep(score, counts)
    for i in range(nb):
        kept = score[i, :i + 1][top[i, :i + 1] == 1]
        dropped = score[i, :i + 1][top[i, :i + 1] == 0]
        assert dropped.size == 0 or kept.min() >= dropped.max()
