"""Host-side checks of the seeded input recipe."""

import math

import numpy as np

import synth


def test_prefill_recipe_structure():
    cfg = synth.CONFIGS["tiny_f32"]
    a = synth.prefill_sequence(cfg.config_seed, 0, cfg.L, cfg.d, cfg.rho, cfg.n_pairs)
    b = synth.prefill_sequence(cfg.config_seed, 0, cfg.L, cfg.d, cfg.rho, cfg.n_pairs)
    for n in ("Q", "K", "V", "dO"):
        assert a[n].shape == (cfg.L, cfg.d)
        assert np.array_equal(a[n], b[n])  # seeded
    c = synth.prefill_sequence(cfg.config_seed, 1, cfg.L, cfg.d, cfg.rho, cfg.n_pairs)
    assert not np.array_equal(a["Q"], c["Q"])  # per-head streams differ
    u = synth.unit_vector(cfg.config_seed, cfg.d)
    assert abs(np.linalg.norm(u) - 1) < 1e-12
    pairs = a["pairs"]
    assert len(pairs) == cfg.n_pairs
    assert len(set(pairs[:, 0])) == len(pairs) and len(set(pairs[:, 1])) == len(pairs)
    for i, j in pairs:
        assert 258 <= i < cfg.L and 1 <= j < i - 256
        qi = a["Q"][i]
        assert np.allclose(a["K"][j], 2.5 * math.sqrt(cfg.d) * qi / np.linalg.norm(qi))
    # sink: K_0 - 6u and Q - 1.5u are the same latent (2.5 x) where no pair landed
    x0k = a["K"][0] - 6 * u
    x0q = a["Q"][0] - 1.5 * u
    assert np.allclose(x0k, x0q)
    # AR(1) latent: lag-1 autocorrelation near rho
    x = (a["Q"] - 1.5 * u) / 2.5
    r = np.sum(x[1:] * x[:-1]) / np.sum(x[:-1] * x[:-1])
    assert abs(r - cfg.rho) < 0.02


def test_decode_recipe_structure():
    cfg = synth.DecodeConfig("small", 4, 2, 8, 2, 4096, 32, 128, 0.98, 16, 4)
    g = synth.decode_group(cfg, 1, 1)
    G = cfg.Hq // cfg.Hkv
    assert g["K"].shape == (cfg.Lc, cfg.d) and g["q"].shape == (G, cfg.d)
    t = g["targets"]
    assert t.shape == (G, cfg.n_query_targets)
    assert len(set(t.ravel())) == t.size and t.max() < cfg.Lc - 256
    for h in range(G):
        for j in t[h]:
            assert np.allclose(g["K"][j], 2.5 * math.sqrt(cfg.d) * g["q"][h] / np.linalg.norm(g["q"][h]))
    full = synth.decode_inputs(cfg, groups=[3])
    assert np.array_equal(full["K"][1, 1], g["K"]) and np.array_equal(full["q"][1, 4:8], g["q"])
