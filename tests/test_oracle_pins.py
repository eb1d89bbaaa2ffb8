"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these compares the oracle with itself: each check uses a library
routine (torch / numpy / scipy), a closed form, a printed example, a
brute-force enumeration or an independent re-derivation.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_inputs(L, d, seed, scale_qk=1.0):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((L, d)) * scale_qk
    K = rng.standard_normal((L, d)) * scale_qk
    V = rng.standard_normal((L, d))
    dO = rng.standard_normal((L, d))
    return Q, K, V, dO


def torch_dense(Q, K, V, dO=None, scale=None):
    """Library reference: torch SDPA (causal, float64) and its autograd."""
    q = torch.tensor(Q, requires_grad=True)
    k = torch.tensor(K, requires_grad=True)
    v = torch.tensor(V, requires_grad=True)
    o = torch.nn.functional.scaled_dot_product_attention(
        q[None, None], k[None, None], v[None, None], is_causal=True, scale=scale)[0, 0]
    out = {"O": o.detach().numpy()}
    if dO is not None:
        o.backward(torch.tensor(dO))
        out.update(dQ=q.grad.numpy(), dK=k.grad.numpy(), dV=v.grad.numpy())
    return out


def causal_scores(Q, K, scale):
    S = scale * (Q @ K.T)
    L = S.shape[0]
    S[np.triu_indices(L, 1)] = -np.inf
    return S


def rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


# --------------------------------------------------------------------------
# tau = 0 is FullAttn (agihunt summary, limits paragraph; gpt-diffusion blog)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("L,d,T", [(1, 4, 4), (37, 8, 8), (130, 16, 32), (200, 16, 64)])
def test_tau0_forward_is_dense_softmax(L, d, T):
    Q, K, V, _ = rand_inputs(L, d, seed=L)
    ref = torch_dense(Q, K, V)
    got = oracle.fwd(Q, K, V, tile=T, tau=0.0)
    assert rel(got["O"], ref["O"]) < 1e-12
    from scipy.special import logsumexp
    lse = logsumexp(causal_scores(Q, K, 1 / math.sqrt(d)), axis=1)
    assert np.max(np.abs(got["LSE"] - lse)) < 1e-12
    nb = oracle.n_blocks(L, T)
    assert np.all(got["keep"][np.tril_indices(nb)] == 1)


@pytest.mark.parametrize("L,d,T", [(37, 8, 8), (130, 16, 32)])
def test_tau0_backward_is_autograd(L, d, T):
    Q, K, V, dO = rand_inputs(L, d, seed=100 + L)
    ref = torch_dense(Q, K, V, dO)
    f = oracle.fwd(Q, K, V, tile=T, tau=0.0)
    g = oracle.bwd(Q, K, V, f["O"], dO, f["LSE"], tile=T, tau=0.0)
    for n in ("dQ", "dK", "dV"):
        assert rel(g[n], ref[n]) < 1e-11, n
    dense = oracle.dense_bwd(Q, K, V, dO)
    for n in ("dQ", "dK", "dV"):
        assert rel(dense[n], ref[n]) < 1e-11, n
    assert rel(oracle.dense_fwd(Q, K, V)["O"], ref["O"]) < 1e-12


def test_tau0_backward_finite_differences():
    """Central differences of the tau=0 forward, L=8, d=4 (no library)."""
    L, d, T = 8, 4, 2
    Q, K, V, dO = rand_inputs(L, d, seed=7)
    f = oracle.fwd(Q, K, V, tile=T, tau=0.0)
    g = oracle.bwd(Q, K, V, f["O"], dO, f["LSE"], tile=T, tau=0.0)
    h = 1e-6

    def loss(Qx, Kx, Vx):
        return float(np.sum(oracle.fwd(Qx, Kx, Vx, tile=T, tau=0.0)["O"] * dO))

    for name, idx in (("dQ", 0), ("dK", 1), ("dV", 2)):
        num = np.zeros((L, d))
        for r in range(L):
            for c in range(d):
                args_p = [Q.copy(), K.copy(), V.copy()]
                args_m = [Q.copy(), K.copy(), V.copy()]
                args_p[idx][r, c] += h
                args_m[idx][r, c] -= h
                num[r, c] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        assert np.max(np.abs(num - g[name])) < 1e-6, name


# --------------------------------------------------------------------------
# Worked example (jaehun.me review, "How it works: a concrete example")
# --------------------------------------------------------------------------
def test_worked_example():
    ex = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    e = np.array(ex["exp_scores_reconstructed"])
    # d = 1, scale = 1, q = 1 at every position, k_c = ln e_c: score(3, c) = ln e_c
    L = 4
    Q = np.ones((L, 1))
    K = np.log(e)[:, None]
    rng = np.random.default_rng(0)
    V = rng.standard_normal((L, 1))  # head dim 1 for q, k and v alike
    f = oracle.fwd(Q, K, V, tile=1, tau=ex["tau"], scale=1.0)
    p = ex["printed"]
    assert ex["tau"] / (ex["query_position"] + 1) == p["threshold"]
    row = f["keep"][3]
    kept = sorted([j for j in range(4) if row[j]], reverse=True)
    assert kept == p["retained_keys"]
    assert sorted(j for j in range(4) if not row[j]) == sorted(p["omitted_keys"])
    # final normalizer: LSE = ln(sum of retained exp-scores)
    assert abs(math.exp(f["LSE"][3]) - p["final_normalizer"]) < 1e-9
    # the k1 ratio exceeds one
    assert e[1] / e[3] > 1.0 and p["ratio_can_exceed_one"]
    # output is softmax renormalised over the retained keys
    f2 = f
    w = e[[3, 1]] / e[[3, 1]].sum()
    assert np.allclose(f2["O"][3], w[0] * V[3] + w[1] * V[1], atol=1e-12)
    # dense mass of each omitted key (~3.4 %) and total omitted (~6.8 %)
    dense = oracle.dense_fwd(Q, K, V, scale=1.0)
    mass = oracle.omitted_mass(Q, K, f["keep"], dense["LSE"], tile=1, scale=1.0)
    assert abs(100 * mass[3] - p["omitted_mass_pct"]) < 0.05
    each = 100 * np.exp(np.log(e[[0, 2]]) - dense["LSE"][3])
    assert np.all(np.abs(each - p["dense_mass_each_omitted_pct"]) < 0.05)
    # backward with the final normalizer keeps {k3, k1}
    dO = rng.standard_normal((L, 1))
    g = oracle.bwd(Q, K, V, f2["O"], dO, f2["LSE"], tile=1, tau=1.0, scale=1.0)
    kept_b = sorted([j for j in range(4) if g["keep"][3, j]], reverse=True)
    assert kept_b == ex["backward_with_final_normalizer"]["retained_keys"]


# --------------------------------------------------------------------------
# Proposition 1 (jaehun.me review, "Theoretical upper bound ...")
# --------------------------------------------------------------------------
@pytest.mark.parametrize("tau", [0.25, 1.0, 4.0, 64.0])
@pytest.mark.parametrize("T", [1, 2, 8])
def test_prop1_bounds(tau, T):
    worst = 0.0
    for seed in range(6):
        L, d = 96, 8
        Q, K, V, _ = rand_inputs(L, d, seed=1000 + seed, scale_qk=1.0 + seed)
        f = oracle.fwd(Q, K, V, tile=T, tau=tau)
        dense = oracle.dense_fwd(Q, K, V)
        mass = oracle.omitted_mass(Q, K, f["keep"], dense["LSE"], tile=T)
        bound = tau / (1 + tau)
        assert np.all(mass <= bound + 1e-12)
        assert np.all(mass >= -1e-12)
        vmax = np.max(np.linalg.norm(V, axis=1))
        err = np.linalg.norm(f["O"] - dense["O"], axis=1)
        assert np.all(err <= 2 * tau / (1 + tau) * vmax + 1e-12)
        worst = max(worst, float(mass.max()))
    # the inputs do exercise skipping
    assert worst > 0.0


def test_every_row_keeps_diagonal_and_is_nonempty():
    L, d, T = 300, 16, 32
    Q, K, V, _ = rand_inputs(L, d, seed=5, scale_qk=3.0)
    for ff in (True, False):
        f = oracle.fwd(Q, K, V, tile=T, tau=1.0, force_first=ff)
        nb = oracle.n_blocks(L, T)
        assert np.all(np.diag(f["keep"]) == 1)
        assert np.all(np.isfinite(f["O"])) and np.all(np.isfinite(f["LSE"]))


# --------------------------------------------------------------------------
# Nesting: backward support within forward support (agihunt summary,
# backward paragraph; jaehun.me review, "Backward: offline ...")
# --------------------------------------------------------------------------
@pytest.mark.parametrize("T", [1, 4, 16])
@pytest.mark.parametrize("tau", [0.5, 1.0, 8.0])
def test_backward_support_nested_in_forward(T, tau):
    L, d = 160, 8
    for seed in range(3):
        Q, K, V, dO = rand_inputs(L, d, seed=2000 + seed, scale_qk=2.0)
        f = oracle.fwd(Q, K, V, tile=T, tau=tau, want_margin=True)
        g = oracle.bwd(Q, K, V, f["O"], dO, f["LSE"], tile=T, tau=tau, want_margin=True)
        nb = oracle.n_blocks(L, T)
        tril = np.tril(np.ones((nb, nb), bool))
        extra = (g["keep"] == 1) & (f["keep"] == 0) & tril
        # exact arithmetic forbids any; allow only ties within rounding
        assert np.all(np.abs(g["margin"][extra]) < 1e-9)
        assert np.sum(extra) == 0
        # backward may drop more (strictly fewer or equal kept tiles)
        assert g["keep"][tril].sum() <= f["keep"][tril].sum()
        # every row keeps at least one tile in backward for tau <= 1
        if tau <= 1.0:
            assert np.all(g["keep"].sum(axis=1) >= 1)


# --------------------------------------------------------------------------
# Brute force: exactly one keep-set is self-consistent with the rule
# --------------------------------------------------------------------------
def consistent_sets(S_block, rows, T, i, tau):
    """All subsets of key tiles j < i (diagonal always in) consistent with the
    sequential test, re-derived directly from the definition: the retained
    normaliser before tile j is the sum over kept tiles visited earlier,
    computed as a plain sum of exponentials (no online update)."""
    found = []
    for bits in itertools.product([0, 1], repeat=i):
        kept = {i} | {j for j in range(i) if bits[j]}
        ok = True
        for j in range(i - 1, -1, -1):
            earlier = [jj for jj in kept if jj > j]
            skip_all = True
            for r in rows:
                vals = [S_block[r][c] for jj in earlier for c in range(jj * T, min((jj + 1) * T, r + 1))]
                z = sum(math.exp(v) for v in vals)
                mt = max(S_block[r][c] for c in range(j * T, (j + 1) * T))
                ratio = math.exp(mt) / z
                if ratio >= tau / (r + 1):
                    skip_all = False
            if (j in kept) == skip_all:
                ok = False
                break
        if ok:
            found.append(kept)
    return found


@pytest.mark.parametrize("T", [1, 2])
def test_bruteforce_keep_sets(T):
    L, d = 12, 3
    for seed in range(4):
        Q, K, V, dO = rand_inputs(L, d, seed=3000 + seed, scale_qk=1.7)
        scale = 1 / math.sqrt(d)
        S = scale * Q @ K.T
        f = oracle.fwd(Q, K, V, tile=T, tau=1.0)
        nb = oracle.n_blocks(L, T)
        for i in range(nb):
            rows = list(range(i * T, min(L, (i + 1) * T)))
            sets = consistent_sets(S, rows, T, i, 1.0)
            assert len(sets) == 1
            assert sets[0] == {j for j in range(i + 1) if f["keep"][i, j]}
            # output = softmax over the retained keys, per row (direct sum)
            for r in rows:
                cols = [c for j in sets[0] for c in range(j * T, min((j + 1) * T, r + 1))]
                w = np.exp(S[r, cols] - S[r, cols].max())
                w /= w.sum()
                assert np.allclose(f["O"][r], w @ V[cols], atol=1e-12)
                assert abs(f["LSE"][r] - np.log(np.sum(np.exp(S[r, cols])))) < 1e-12


def test_backward_matches_masked_matrix_gradients():
    """Backward on kept tiles re-derived in matrix form with numpy."""
    L, d, T = 64, 8, 4
    Q, K, V, dO = rand_inputs(L, d, seed=11, scale_qk=3.0)
    scale = 1 / math.sqrt(d)
    f = oracle.fwd(Q, K, V, tile=T, tau=1.0)
    g = oracle.bwd(Q, K, V, f["O"], dO, f["LSE"], tile=T, tau=1.0)
    mask = np.kron(g["keep"], np.ones((T, T)))[:L, :L].astype(bool)
    mask &= np.tril(np.ones((L, L), bool))
    P = np.where(mask, np.exp(scale * Q @ K.T - f["LSE"][:, None]), 0.0)
    Dv = np.sum(dO * f["O"], axis=1)
    dP = dO @ V.T
    dS = P * (dP - Dv[:, None])
    assert rel(g["dV"], P.T @ dO) < 1e-12
    assert rel(g["dQ"], scale * dS @ K) < 1e-12
    assert rel(g["dK"], scale * dS.T @ Q) < 1e-12
    # and some tiles were actually dropped
    assert g["keep"][np.tril_indices(L // T)].min() == 0


def test_partial_block_ranges_match_full():
    L, d, T = 100, 8, 16
    Q, K, V, dO = rand_inputs(L, d, seed=12, scale_qk=2.0)
    full = oracle.fwd(Q, K, V, tile=T)
    part = oracle.fwd(Q, K, V, tile=T, qblocks=(3, 5))
    assert np.array_equal(part["O"][48:80], full["O"][48:80])
    assert np.array_equal(part["keep"][3:5], full["keep"][3:5])
    gb = oracle.bwd(Q, K, V, full["O"], dO, full["LSE"], tile=T)
    gp = oracle.bwd(Q, K, V, full["O"], dO, full["LSE"], tile=T, qblocks=[6], kblocks=[2, 6])
    assert np.allclose(gp["dQ"][96:], gb["dQ"][96:], rtol=0, atol=1e-13)
    assert np.allclose(gp["dK"][32:48], gb["dK"][32:48], rtol=0, atol=1e-13)
    assert np.allclose(gp["dV"][96:], gb["dV"][96:], rtol=0, atol=1e-13)


# --------------------------------------------------------------------------
# Invariance: a per-row constant added to every score changes nothing
# --------------------------------------------------------------------------
def test_row_shift_invariance():
    L, d, T = 96, 8, 16
    Q, K, V, dO = rand_inputs(L, d, seed=13, scale_qk=2.0)
    w = np.random.default_rng(1).standard_normal(d)
    a = oracle.fwd(Q, K, V, tile=T, tau=1.0)
    b = oracle.fwd(Q, K + w, V, tile=T, tau=1.0)  # row r shifts by scale*<q_r, w>
    assert np.array_equal(a["keep"], b["keep"])
    assert rel(b["O"], a["O"]) < 1e-12


# --------------------------------------------------------------------------
# Decode (one rule for prefill and decode; agihunt summary, rule paragraph)
# --------------------------------------------------------------------------
def test_decode_equals_prefill_last_row():
    """With one query head per KV head and Lc = n*T + 1, the decode tiles are
    exactly the prefill tiles seen by the last (single-row) query block."""
    T, n, d = 8, 9, 8
    Lc = n * T + 1
    Q, K, V, _ = rand_inputs(Lc, d, seed=21, scale_qk=2.0)
    f = oracle.fwd(Q, K, V, tile=T, tau=1.0)
    dec = oracle.decode(Q[-1:], K[None], V[None], tau=1.0, tile=T)
    assert np.allclose(dec["o"][0], f["O"][-1], rtol=0, atol=1e-13)
    assert np.array_equal(dec["keep"][0], f["keep"][n])


def test_decode_tau0_is_softmax():
    Hq, Hkv, Lc, d = 8, 2, 300, 16
    rng = np.random.default_rng(22)
    q = rng.standard_normal((Hq, d))
    Kc = rng.standard_normal((Hkv, Lc, d))
    Vc = rng.standard_normal((Hkv, Lc, d))
    dec = oracle.decode(q, Kc, Vc, tau=0.0, tile=128)
    for h in range(Hq):
        g = h // (Hq // Hkv)
        p = torch.softmax(torch.tensor(q[h] @ Kc[g].T / math.sqrt(d)), 0).numpy()
        assert np.allclose(dec["o"][h], p @ Vc[g], rtol=0, atol=1e-12)


def test_decode_group_rows():
    """Group rows: a tile is kept when any head of the KV group passes; with
    one head per group this is the per-head rule; Proposition 1 holds for
    every head."""
    Hq, Hkv, Lc, d = 8, 2, 2000, 16
    rng = np.random.default_rng(23)
    q = rng.standard_normal((Hq, d)) * 2.5
    Kc = rng.standard_normal((Hkv, Lc, d)) * 2.5
    Vc = rng.standard_normal((Hkv, Lc, d))
    G = Hq // Hkv
    grp = oracle.decode(q, Kc, Vc, tau=1.0, tile=64)
    ph = oracle.decode(q, Kc, Vc, tau=1.0, tile=64, per_head=True)
    one = oracle.decode(q[:Hkv], Kc, Vc, tau=1.0, tile=64)
    one_ph = oracle.decode(q[:Hkv], Kc, Vc, tau=1.0, tile=64, per_head=True)
    assert np.array_equal(one["keep"], one_ph["keep"])
    assert np.allclose(one["o"], one_ph["o"], rtol=0, atol=0)
    assert grp["keep"].sum() < grp["keep"].size  # something skipped
    assert ph["keep"].sum() < ph["keep"].size
    for h in range(Hq):
        g = h // G
        s = q[h] @ Kc[g].T / math.sqrt(d)
        lse = np.log(np.sum(np.exp(s - s.max()))) + s.max()
        kept_cols = np.repeat(grp["keep"][g], 64)[:Lc].astype(bool)
        omitted = 1 - np.sum(np.exp(s[kept_cols] - lse))
        assert omitted <= 0.5 + 1e-12
        w = np.exp(s[kept_cols] - s[kept_cols].max())
        assert np.allclose(grp["o"][h], (w / w.sum()) @ Vc[g][kept_cols], rtol=0, atol=1e-12)


def decode_consistent_sets(S, T, tau):
    """All subsets of a cache's key tiles (the newest always in) consistent
    with the sequential decode test, re-derived from the definition: rows are
    the heads in S ([rows][Lc] scores), a tile is kept when any row's ratio
    exp(tile max) / (sum of exp over the kept tiles visited earlier) reaches
    tau / Lc; plain sums, no online update."""
    Lc = len(S[0])
    nt = -(-Lc // T)
    found = []
    for bits in itertools.product([0, 1], repeat=nt - 1):
        kept = {nt - 1} | {t for t in range(nt - 1) if bits[t]}
        ok = True
        for t in range(nt - 2, -1, -1):
            earlier = [tt for tt in kept if tt > t]
            keep_t = False
            for s in S:
                z = sum(math.exp(s[c]) for tt in earlier for c in range(tt * T, min((tt + 1) * T, Lc)))
                mt = max(s[c] for c in range(t * T, min((t + 1) * T, Lc)))
                if math.exp(mt) / z >= tau / Lc:
                    keep_t = True
            if (t in kept) != keep_t:
                ok = False
                break
        if ok:
            found.append(kept)
    return found


@pytest.mark.parametrize("T", [1, 2])
def test_decode_bruteforce_keep_sets(T):
    """Tiny caches: exactly one keep set per KV group (group rows) and per head
    (per-head rows) is consistent with the sequential rule, it is the
    oracle's, and each head's output is the softmax over the kept keys."""
    Hq, Hkv, Lc, d, tau = 6, 2, 11, 3, 1.0
    G = Hq // Hkv
    nt = -(-Lc // T)
    skipped = kept_old = 0
    for seed in range(3):
        rng = np.random.default_rng(5100 + seed)
        q = rng.standard_normal((Hq, d)) * 1.8
        Kc = rng.standard_normal((Hkv, Lc, d)) * 1.8
        Vc = rng.standard_normal((Hkv, Lc, d))
        S = [q[h] @ Kc[h // G].T / math.sqrt(d) for h in range(Hq)]
        for per_head in (False, True):
            out = oracle.decode(q, Kc, Vc, tau=tau, tile=T, per_head=per_head)
            for u in range(Hq if per_head else Hkv):
                heads = [u] if per_head else list(range(u * G, (u + 1) * G))
                sets = decode_consistent_sets([S[h] for h in heads], T, tau)
                assert len(sets) == 1
                assert sets[0] == {t for t in range(nt) if out["keep"][u, t]}
                skipped += nt - len(sets[0])
                kept_old += len(sets[0]) - 1
                for h in heads:
                    cols = [c for t in sets[0] for c in range(t * T, min((t + 1) * T, Lc))]
                    w = np.exp(S[h][cols] - S[h][cols].max())
                    assert np.allclose(out["o"][h], (w / w.sum()) @ Vc[h // G][cols], rtol=0,
                                       atol=1e-12)
    assert skipped > 0 and kept_old > 0  # both branches of the test were taken


def test_decode_head_permutation():
    """Permuting the query heads inside each KV group leaves the group's keep
    set unchanged and permutes the outputs; permuting the KV groups together
    with their query heads permutes both."""
    Hq, Hkv, Lc, d = 8, 2, 700, 16
    G = Hq // Hkv
    rng = np.random.default_rng(29)
    q = rng.standard_normal((Hq, d)) * 2.5
    Kc = rng.standard_normal((Hkv, Lc, d)) * 2.5
    Vc = rng.standard_normal((Hkv, Lc, d))
    base = oracle.decode(q, Kc, Vc, tau=1.0, tile=32)
    assert 0 < base["keep"].sum() < base["keep"].size
    inner = np.concatenate([g * G + rng.permutation(G) for g in range(Hkv)])
    p = oracle.decode(q[inner], Kc, Vc, tau=1.0, tile=32)
    assert np.array_equal(p["keep"], base["keep"])
    assert np.array_equal(p["o"], base["o"][inner])
    gp = np.array([1, 0])
    heads = np.concatenate([np.arange(g * G, (g + 1) * G) for g in gp])
    p = oracle.decode(q[heads], Kc[gp], Vc[gp], tau=1.0, tile=32)
    assert np.array_equal(p["keep"], base["keep"][gp])
    assert np.array_equal(p["o"], base["o"][heads])


@pytest.mark.parametrize("tau,T", [(1.0, 8), (0.25, 8), (4.0, 4), (0.0, 8)])
def test_forward_from_maxima_then_scan_then_pv(tau, T):
    """The forward's rule re-derived in another order (numpy): every legal
    tile's row maxima first; then, per query block, the sequential test on
    those maxima alone, a kept tile's row sums exp(S - max) taken from its
    scores only when it is kept; then O = sum over kept tiles of
    exp(S - m) V / l with the final (m, l). It must give the oracle's keep
    set, LSE and output."""
    L, d = 203, 8
    Q, K, V, _ = rand_inputs(L, d, 61, scale_qk=2.5)
    scale = 1.0 / math.sqrt(d)
    S = scale * Q @ K.T
    S[np.triu(np.ones((L, L), bool), 1)] = -np.inf
    nb = oracle.n_blocks(L, T)
    f = oracle.fwd(Q, K, V, tile=T, tau=tau)
    O = np.zeros((L, d))
    LSE = np.zeros(L)
    for i in range(nb):
        rows = np.arange(i * T, min(L, (i + 1) * T))
        tiles = [np.arange(j * T, min(L, (j + 1) * T)) for j in range(i + 1)]
        mt = [S[np.ix_(rows, c)].max(axis=1) for c in tiles]        # phase A
        m = np.full(len(rows), -np.inf)
        l = np.zeros(len(rows))
        kept = []
        for j in range(i, -1, -1):                                    # phase B
            if j != i and tau > 0:
                lhs = mt[j] - m - np.log(l)
                if np.all(lhs < math.log(tau) - np.log(rows + 1)):
                    continue
            kept.append(j)
            lt = np.exp(S[np.ix_(rows, tiles[j])] - mt[j][:, None]).sum(axis=1)
            mn = np.maximum(m, mt[j])
            l = l * np.exp(m - mn) + lt * np.exp(mt[j] - mn)
            m = mn
        assert sorted(kept) == [j for j in range(i + 1) if f["keep"][i, j]]
        cols = np.concatenate([tiles[j] for j in kept])               # phase C
        P = np.exp(S[np.ix_(rows, cols)] - m[:, None])
        O[rows] = P @ V[cols] / l[:, None]
        LSE[rows] = m + np.log(l)
    assert np.allclose(LSE, f["LSE"], rtol=0, atol=1e-12)
    assert np.allclose(O, f["O"], rtol=0, atol=1e-12)
    if tau > 0:
        assert f["keep"][np.tril_indices(nb)].min() == 0  # something was skipped


def test_tile_row_max_bruteforce():
    """Pure-Python enumeration of every (row, legal key) score on a tiny
    ragged case (L = 7, tile 3: blocks of 3, 3, 1 rows)."""
    rng = np.random.default_rng(41)
    L, d, T = 7, 2, 3
    Q, K = rng.standard_normal((L, d)), rng.standard_normal((L, d))
    got = oracle.tile_row_max(Q, K, T)
    assert sorted(got) == [0, 1, 2]
    for i in range(3):
        for j in range(i + 1):
            for r in range(T):
                row = i * T + r
                if row >= L:
                    assert got[i][j, r] == -np.inf
                    continue
                best = -math.inf
                for c in range(j * T, min(L, (j + 1) * T)):
                    if c <= row:
                        best = max(best, sum(Q[row, e] * K[c, e] for e in range(d)))
                assert got[i][j, r] == pytest.approx(best, abs=1e-12)


@pytest.mark.parametrize("tau", [1.0, 0.25])
def test_tile_row_max_decides_the_backward_keep_set(tau):
    """The backward's keep set follows from the tile row maxima and the final
    LSE alone: tile (i, j) stays iff some valid row has
    scale * max >= LSE + ln tau - ln(row + 1)."""
    L, d, T = 300, 8, 8
    Q, K, V, dO = rand_inputs(L, d, 43, scale_qk=3.0)
    scale = 1.0 / math.sqrt(d)
    f = oracle.fwd(Q, K, V, tile=T, tau=tau)
    g = oracle.bwd(Q, K, V, f["O"], dO, f["LSE"], tile=T, tau=tau, want_margin=True)
    rm = oracle.tile_row_max(Q, K, T)
    nb = oracle.n_blocks(L, T)
    skipped = 0
    for i in range(nb):
        for j in range(i + 1):
            rows = np.arange(i * T, min(L, (i + 1) * T))
            margin = scale * rm[i][j, :len(rows)] - (f["LSE"][rows] + math.log(tau) - np.log(rows + 1))
            assert int(margin.max() >= 0) == g["keep"][i, j], (i, j)
            assert margin.max() == pytest.approx(g["margin"][i, j], abs=1e-9)
            skipped += int(g["keep"][i, j] == 0)
    assert skipped > 0


@pytest.mark.parametrize("tau", [0.5, 1.0, 4.0])
def test_omitted_mass_from_two_log_normalizers(tau):
    """The mass a query row loses to skipped tiles equals 1 - exp(LSE_tau -
    LSE_dense): LSE_tau normalizes over the kept keys only (the forward's
    output), LSE_dense over all legal keys (tau = 0). Checked against the
    per-tile enumeration of omitted_mass."""
    L, d, T = 300, 8, 8
    Q, K, V, _ = rand_inputs(L, d, 51, scale_qk=3.0)
    f = oracle.fwd(Q, K, V, tile=T, tau=tau)
    dense = oracle.fwd(Q, K, V, tile=T, tau=0.0)
    mass = oracle.omitted_mass(Q, K, f["keep"], dense["LSE"], tile=T)
    np.testing.assert_allclose(mass, 1.0 - np.exp(f["LSE"] - dense["LSE"]), atol=1e-12)
    assert mass.max() > 0
    assert mass.max() <= tau / (1 + tau) + 1e-12


def test_grouped_heads_backward_sums_over_the_group():
    """Grouped query heads (several query heads read one key/value head): the
    forward is the per-head rule on the shared K, V, and dK, dV of the shared
    head are the sums of the per-head gradients. At tau = 0 this is checked
    against torch autograd through K, V repeated for every query head (the
    repeat's backward does the summing)."""
    rng = np.random.default_rng(61)
    G, L, d, T = 3, 40, 8, 8
    K, V = rng.standard_normal((L, d)), rng.standard_normal((L, d))
    Qs = [rng.standard_normal((L, d)) * 1.3 for _ in range(G)]
    dOs = [rng.standard_normal((L, d)) for _ in range(G)]
    dK, dV = np.zeros((L, d)), np.zeros((L, d))
    outs = []
    for Q, dO in zip(Qs, dOs):
        f = oracle.fwd(Q, K, V, tile=T, tau=0.0)
        g = oracle.bwd(Q, K, V, f["O"], dO, f["LSE"], tile=T, tau=0.0)
        dK += g["dK"]
        dV += g["dV"]
        outs.append((f["O"], g["dQ"]))
    q = torch.tensor(np.stack(Qs), requires_grad=True)
    k = torch.tensor(K, requires_grad=True)
    v = torch.tensor(V, requires_grad=True)
    o = torch.nn.functional.scaled_dot_product_attention(
        q[None], k[None, None].expand(1, G, L, d), v[None, None].expand(1, G, L, d),
        is_causal=True)[0]
    o.backward(torch.tensor(np.stack(dOs)))
    for h, (O, dQ) in enumerate(outs):
        np.testing.assert_allclose(O, o[h].detach().numpy(), atol=1e-10)
        np.testing.assert_allclose(dQ, q.grad[h].numpy(), atol=1e-9)
    np.testing.assert_allclose(dK, k.grad.numpy(), atol=1e-9)
    np.testing.assert_allclose(dV, v.grad.numpy(), atol=1e-9)


@pytest.mark.parametrize("off", [0, 16, 24, 5])
def test_chunk_forward_dense_is_bottom_right_causal_softmax(off):
    """tau = 0: a chunk of Lq queries after `off` cached keys is softmax
    attention where query r sees keys 0 .. off + r (library: torch SDPA with
    that mask, float64)."""
    rng = np.random.default_rng(71 + off)
    Lq, d, T = 37, 8, 8
    Lk = Lq + off
    Q, K, V = (rng.standard_normal((n, d)) for n in (Lq, Lk, Lk))
    f = oracle.fwd_chunk(Q, K, V, tile=T, tau=0.0)
    mask = np.arange(Lk)[None, :] <= (off + np.arange(Lq))[:, None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(Q)[None, None], torch.tensor(K)[None, None], torch.tensor(V)[None, None],
        attn_mask=torch.tensor(mask)[None, None])[0, 0].numpy()
    np.testing.assert_allclose(f["O"], ref, atol=1e-12)


@pytest.mark.parametrize("tau", [0.5, 1.0, 4.0])
def test_chunk_forward_equals_full_prefill_rows(tau):
    """A chunk whose cache length is a multiple of the tile sees exactly the
    tiles and running state of the full prefill's last blocks, so it
    reproduces their outputs, log-normalizers and keep sets."""
    L, d, T = 160, 8, 16
    Q, K, V, _ = rand_inputs(L, d, 73, scale_qk=2.5)
    for off in (0, 48, 96):
        full = oracle.fwd(Q, K, V, tile=T, tau=tau)
        ch = oracle.fwd_chunk(Q[off:], K, V, tile=T, tau=tau)
        np.testing.assert_allclose(ch["O"], full["O"][off:], atol=1e-12)
        np.testing.assert_allclose(ch["LSE"], full["LSE"][off:], atol=1e-12)
        b0 = off // T
        assert np.array_equal(ch["keep"], full["keep"][b0:, :])


def test_chunk_forward_keeps_the_mass_bound():
    """Any cache offset: the mass a row loses stays below tau / (1 + tau)."""
    rng = np.random.default_rng(79)
    Lq, d, T, off, tau = 70, 8, 8, 29, 1.0
    Q, K, V = (rng.standard_normal((n, d)) * 2.5 for n in (Lq, Lq + off, Lq + off))
    f = oracle.fwd_chunk(Q, K, V, tile=T, tau=tau)
    dense = oracle.fwd_chunk(Q, K, V, tile=T, tau=0.0)
    lost = 1.0 - np.exp(f["LSE"] - dense["LSE"])
    assert lost.max() > 0 and lost.max() <= tau / (1 + tau)
    assert f["keep"].sum() < dense["keep"].sum()
