"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs. Every test here needs a B200 and the built library."""

from __future__ import annotations


import numpy as np
import pytest

import oracle
import synth
from tests.parity import (TOL, Coverage, as_f64, compare_bwd_keep, compare_decode_keep,
                          compare_fwd_keep, grad_row_masks, rel_l2, row_mask)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU container
    pytest.skip("needs a GPU", allow_module_level=True)

import mass_adaptive_causal_b200 as mala  # noqa: E402


def dev_tensor(a, dtype):
    return torch.tensor(np.ascontiguousarray(a), dtype=torch.float64).to(dtype).cuda()


def rounded(t):
    """The exact values the GPU sees (bf16/f32 -> float64)."""
    return as_f64(t)


def prefill_case(cfg, L=None, heads=None, dtype=torch.bfloat16):
    x = synth.prefill_inputs(cfg, L=L, heads=heads)
    t = {n: dev_tensor(x[n], dtype) for n in ("Q", "K", "V", "dO")}
    return t


def check_fwd_slice(Qd, Kd, Vd, O_gpu, LSE_gpu, bits_gpu, tile, tau, tol, qblocks=None,
                    cov=None):
    """One (b, h) slice; returns (rows_compared, near_flips, oracle result,
    query blocks with an allowed flip)."""
    L = Qd.shape[0]
    nb = oracle.n_blocks(L, tile)
    ref = oracle.fwd(Qd, Kd, Vd, tile=tile, tau=tau, want_margin=True, qblocks=qblocks)
    lo, hi = (0, nb) if qblocks is None else qblocks
    gk = mala.unpack_bits(bits_gpu, nb)
    n_near, bad = compare_fwd_keep(gk[lo:hi], ref["keep"][lo:hi], ref["margin"][lo:hi], lo)
    bad = [b + lo for b in bad]
    rows = row_mask(L, tile, bad)
    sel = np.zeros(L, bool)
    sel[lo * tile:min(L, hi * tile)] = True
    rows &= sel
    if rows.any():
        assert rel_l2(O_gpu[rows], ref["O"][rows]) <= tol["O"]
        assert rel_l2(LSE_gpu[rows], ref["LSE"][rows]) <= tol["LSE"]
    if cov is not None:
        cov.add("O", rows[sel])
        cov.flips["fwd"] += n_near
        cov.slices += 1
    return int(rows.sum()), n_near, ref, bad


# ----------------------------------------------------------------------------
# float32 path (64 x 64 tiles)
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("tau", [1.0, 0.0])
def test_f32_tiny_config_fwd_bwd(tau):
    """B=1 H=1 L=1024 d=64 float32, tile 64: the tiny configuration."""
    cfg = synth.CONFIGS["tiny_f32"]
    t = prefill_case(cfg, dtype=torch.float32)
    O, LSE, kept, bits = mala.mala_fwd(t["Q"], t["K"], t["V"], tau=tau, trace=True)
    dQ, dK, dV, kept_b, bits_b = mala.mala_bwd(t["Q"], t["K"], t["V"], O, t["dO"], LSE, tau=tau,
                                               trace=True)
    mala.mala_check()
    Qd, Kd, Vd, dOd = (rounded(t[n][0, 0]) for n in ("Q", "K", "V", "dO"))
    _, n_near, ref, _ = check_fwd_slice(Qd, Kd, Vd, as_f64(O[0, 0]), as_f64(LSE[0, 0]),
                                        bits[0, 0], 64, tau, TOL["f32"])
    assert n_near == 0
    nb = 16
    assert np.array_equal(kept[0, 0].cpu().numpy(), ref["keep"].sum(axis=1))
    g = oracle.bwd(Qd, Kd, Vd, ref["O"], dOd, ref["LSE"], tile=64, tau=tau, want_margin=True)
    assert compare_bwd_keep(mala.unpack_bits(bits_b[0, 0], nb), g["keep"], g["margin"]) == []
    assert np.array_equal(kept_b[0, 0].cpu().numpy(), g["keep"].sum(axis=0))
    for n, a in (("dQ", dQ), ("dK", dK), ("dV", dV)):
        assert rel_l2(as_f64(a[0, 0]), g[n]) <= TOL["f32"]["grad"], n
    if tau == 0.0:
        dense = oracle.dense_fwd(Qd, Kd, Vd)
        assert rel_l2(as_f64(O[0, 0]), dense["O"]) <= 1e-5


@pytest.mark.parametrize("L,d,B,H", [(1, 64, 1, 1), (63, 32, 2, 1), (65, 64, 1, 3),
                                     (200, 128, 2, 2), (512, 64, 1, 1)])
def test_f32_ragged_shapes(L, d, B, H):
    rng = np.random.default_rng(L * 7 + d)
    Q = rng.standard_normal((B, H, L, d)) * 2.0
    K = rng.standard_normal((B, H, L, d)) * 2.0
    V = rng.standard_normal((B, H, L, d))
    dO = rng.standard_normal((B, H, L, d))
    t = {n: dev_tensor(a, torch.float32) for n, a in zip(("Q", "K", "V", "dO"), (Q, K, V, dO))}
    O, LSE, kept, bits = mala.mala_fwd(t["Q"], t["K"], t["V"], tau=1.0, trace=True)
    dQ, dK, dV = mala.mala_bwd(t["Q"], t["K"], t["V"], O, t["dO"], LSE, tau=1.0)
    mala.mala_check()
    for b in range(B):
        for h in range(H):
            Qd, Kd, Vd, dOd = (rounded(t[n][b, h]) for n in ("Q", "K", "V", "dO"))
            _, n_near, ref, _ = check_fwd_slice(Qd, Kd, Vd, as_f64(O[b, h]), as_f64(LSE[b, h]),
                                                bits[b, h], 64, 1.0, TOL["f32"])
            assert n_near == 0
            g = oracle.bwd(Qd, Kd, Vd, ref["O"], dOd, ref["LSE"], tile=64, tau=1.0)
            for n, a in (("dQ", dQ), ("dK", dK), ("dV", dV)):
                assert rel_l2(as_f64(a[b, h]), g[n]) <= TOL["f32"]["grad"], n


# ----------------------------------------------------------------------------
# bf16 tcgen05 path (128 x 128 tiles, d = 128)
# ----------------------------------------------------------------------------
def run_bf16_prefill(t, tau, use_o32=True):
    """The training chain: forward (with its float32 output when use_o32),
    then backward; only O (or its float32 copy) and LSE pass between them."""
    O, LSE, kept, bits, *rest = mala.mala_fwd(t["Q"], t["K"], t["V"], tau=tau, trace=True,
                                              o32=use_o32)
    o32 = rest[0] if use_o32 else None
    dQ, dK, dV, kept_b, bits_b = mala.mala_bwd(t["Q"], t["K"], t["V"], O, t["dO"], LSE, tau=tau,
                                               trace=True, o32=o32)
    mala.mala_check()
    if use_o32:  # the float32 output is the bf16 output before rounding
        assert torch.equal(o32.to(torch.bfloat16), O)
    return O, LSE, kept, bits, dQ, dK, dV, kept_b, bits_b


def bf16_round(a):
    return torch.tensor(a).to(torch.bfloat16).double().numpy()


def check_bf16_slice(t, outs, b, h, tau, cov, grads=True, o_rounded=False):
    """Forward against the oracle; backward against the oracle's backward fed
    the oracle's own forward output. With ``o_rounded`` (the chain without
    the float32 output) the backward's row terms D_r = <dO_r, O_r> are
    defined on the bf16 O it is given, so the oracle is fed its own O rounded
    to bf16. Rows touched by an allowed near-threshold flip are left out
    (tests/parity.py); ``cov`` records what was compared."""
    O, LSE, kept, bits, dQ, dK, dV, kept_b, bits_b = outs
    Qd, Kd, Vd, dOd = (rounded(t[n][b, h]) for n in ("Q", "K", "V", "dO"))
    L = Qd.shape[0]
    nb = oracle.n_blocks(L, 128)
    _, _, ref, bad = check_fwd_slice(Qd, Kd, Vd, as_f64(O[b, h]), as_f64(LSE[b, h]), bits[b, h],
                                     128, tau, TOL["bf16"], cov=cov)
    if not bad:
        assert np.array_equal(kept[b, h].cpu().numpy(), ref["keep"].sum(axis=1))
    if not grads:
        return
    O_in = bf16_round(ref["O"]) if o_rounded else ref["O"]
    g = oracle.bwd(Qd, Kd, Vd, O_in, dOd, ref["LSE"], tile=128, tau=tau, want_margin=True)
    gb = mala.unpack_bits(bits_b[b, h], nb)
    flips = compare_bwd_keep(gb, g["keep"], g["margin"], skip_blocks=bad)
    cov.flips["bwd"] += len(flips)
    qmask, kmask = grad_row_masks(L, 128, bad, flips, gb, g["keep"])
    for n, a, m in (("dQ", dQ, qmask), ("dK", dK, kmask), ("dV", dV, kmask)):
        if m.any():
            assert rel_l2(as_f64(a[b, h])[m], g[n][m]) <= TOL["bf16"]["grad"], n
        cov.add(n, m)


@pytest.mark.parametrize("L", [128, 1000, 1536])
@pytest.mark.parametrize("tau", [1.0, 0.0])
def test_bf16_small_fwd_bwd(L, tau):
    cfg = synth.CONFIGS["matched_8k"]
    t = prefill_case(cfg, L=L, heads=[0, 1])
    t = {n: v[:, :2].contiguous() for n, v in t.items()}
    outs = run_bf16_prefill(t, tau)
    cov = Coverage(f"small L={L} tau={tau}")
    for h in range(2):
        check_bf16_slice(t, outs, 0, h, tau, cov)
    cov.require(0.5)


def test_bf16_backward_column_starting_below_its_diagonal():
    """On random inputs at tau = 32 some key columns fail the backward's test
    on their diagonal tile while later query blocks keep them, so a column's
    first kept tile is not the diagonal one (the work pass then drops its
    early copies of the diagonal block): the gradients still follow the
    oracle."""
    rng = np.random.default_rng(11)
    L, tau = 2048, 32.0
    arrs = [rng.standard_normal((1, 2, L, 128)) for _ in range(4)]
    t = {n: dev_tensor(a, torch.bfloat16) for n, a in zip(("Q", "K", "V", "dO"), arrs)}
    outs = run_bf16_prefill(t, tau)
    nb = oracle.n_blocks(L, 128)
    gb = mala.unpack_bits(outs[8][0], nb)  # (heads, nb, nb) backward keep bits
    assert sum(1 for h in range(2) for j in range(nb) if gb[h, j, j] == 0 and gb[h, j + 1:, j].any()) > 0
    cov = Coverage(f"column below its diagonal tau={tau}")
    for h in range(2):
        check_bf16_slice(t, outs, 0, h, tau, cov)
    cov.require(0.5)


@pytest.mark.parametrize("L", [1000])
def test_bf16_chain_without_float32_output(L):
    """Backward with D from the bf16 output (no float32 copy)."""
    cfg = synth.CONFIGS["matched_8k"]
    t = prefill_case(cfg, L=L, heads=[0, 1])
    t = {n: v[:, :2].contiguous() for n, v in t.items()}
    outs = run_bf16_prefill(t, 1.0, use_o32=False)
    cov = Coverage("chain without float32 output")
    for h in range(2):
        check_bf16_slice(t, outs, 0, h, 1.0, cov, o_rounded=True)
    cov.require(0.5)


def test_bf16_random_inputs_multi_batch():
    rng = np.random.default_rng(5)
    B, H, L, d = 2, 2, 700, 128
    arrs = [rng.standard_normal((B, H, L, d)) * s for s in (1.5, 1.5, 1.0, 1.0)]
    t = {n: dev_tensor(a, torch.bfloat16) for n, a in zip(("Q", "K", "V", "dO"), arrs)}
    outs = run_bf16_prefill(t, 1.0)
    cov = Coverage("random inputs B=2 H=2")
    for b in range(B):
        for h in range(H):
            check_bf16_slice(t, outs, b, h, 1.0, cov)
    cov.require(0.5)


def test_bf16_matched_work_config_full():
    """B=1 H=8 L=8192 d=128 bf16 tile 128 tau=1: every head, every output."""
    cfg = synth.CONFIGS["matched_8k"]
    t = prefill_case(cfg)
    outs = run_bf16_prefill(t, 1.0)
    cov = Coverage("matched_8k")
    for h in range(cfg.H):
        check_bf16_slice(t, outs, 0, h, 1.0, cov)
    cov.require(0.75)


@pytest.mark.parametrize("L", [1024, 2048, 4096, 8192])
@pytest.mark.parametrize("tau", [1.0, 0.0])
def test_bf16_sweep_config_all_heads(L, tau):
    """Length-sweep configuration (B=1 H=16 d=128 bf16 tile 128) at the
    lengths up to 8K: forward and backward of all 16 heads."""
    cfg = synth.CONFIGS[f"sweep_L{L}"]
    t = prefill_case(cfg)
    outs = run_bf16_prefill(t, tau)
    cov = Coverage(f"sweep L={L} tau={tau}")
    for h in range(cfg.H):
        check_bf16_slice(t, outs, 0, h, tau, cov)
    cov.require(0.75)


@pytest.mark.parametrize("tau", [1.0, 0.0])
def test_bf16_sweep_16k_two_heads(tau):
    """Length-sweep configuration at L=16384 (H=16): heads 0 and 9, forward
    and backward."""
    cfg = synth.CONFIGS["sweep_L16384"]
    t = prefill_case(cfg, heads=[0, 9])
    outs = run_bf16_prefill(t, tau)
    cov = Coverage(f"sweep L=16384 tau={tau}")
    for h in range(2):
        check_bf16_slice(t, outs, 0, h, tau, cov)
    cov.require(0.75)


# ----------------------------------------------------------------------------
# decode
# ----------------------------------------------------------------------------
def check_decode(q, Kc, Vc, o, kept, bits, tau, groups, min_frac=0.75):
    """Keep sets, kept counts and outputs of the given (b, kv head) groups. A
    group with an allowed near-threshold flip is counted, not compared (its
    heads share the decisions, so its whole output legitimately differs); at
    least ``min_frac`` of the groups must be compared."""
    B, Hq, d = q.shape
    Hkv, Lc = Kc.shape[1], Kc.shape[2]
    G = Hq // Hkv
    nt = oracle.n_blocks(Lc, 128)
    cov = Coverage(f"decode B={B} Hq={Hq} Hkv={Hkv} Lc={Lc} tau={tau}")
    for b in sorted(set(g // Hkv for g in groups)):
        ref = oracle.decode(rounded(q[b]), rounded(Kc[b]), rounded(Vc[b]), tau=tau,
                            want_margin=True)
        gk = mala.unpack_bits(bits[b], nt)
        for g in range(Hkv):
            if b * Hkv + g not in groups:
                continue
            cov.slices += 1
            if compare_decode_keep(gk[g], ref["keep"][g], ref["margin"][g]):
                cov.flips["decode"] += 1
                cov.add("o", np.zeros(G, bool))
                continue
            assert kept[b, g].item() == int(ref["keep"][g].sum())
            sl = slice(g * G, (g + 1) * G)
            assert rel_l2(as_f64(o[b, sl]), ref["o"][sl]) <= TOL["bf16"]["decode"]
            cov.add("o", np.ones(G, bool))
    cov.require(min_frac)


def test_decode_long_cache_wraps_the_ring():
    """4 groups x 1024 tiles: every CTA of the streaming pass cycles its TMA
    ring several times."""
    cfg = synth.DecodeConfig("wrap", 4, 2, 8, 2, 131072, 128, 128, 0.98, 1024, 4)
    x = synth.decode_inputs(cfg)
    q = dev_tensor(x["q"], torch.bfloat16)
    Kc = dev_tensor(x["K"], torch.bfloat16)
    Vc = dev_tensor(x["V"], torch.bfloat16)
    for _ in range(2):
        o, kept, bits = mala.mala_decode(q, Kc, Vc, tau=1.0, trace=True)
    mala.mala_check()
    check_decode(q, Kc, Vc, o, kept, bits, 1.0, set(range(cfg.B * cfg.Hkv)))


@pytest.mark.parametrize("Lc", [1, 127, 128, 1000, 5000])
@pytest.mark.parametrize("tau", [1.0, 0.0])
def test_decode_small(Lc, tau):
    cfg = synth.DecodeConfig("small", 4, 2, 8, 2, Lc, 128, 128, 0.98, max(0, Lc // 256), 4 if Lc > 300 else 0)
    x = synth.decode_inputs(cfg)
    q = dev_tensor(x["q"], torch.bfloat16)
    Kc = dev_tensor(x["K"], torch.bfloat16)
    Vc = dev_tensor(x["V"], torch.bfloat16)
    o, kept, bits = mala.mala_decode(q, Kc, Vc, tau=tau, trace=True)
    mala.mala_check()
    check_decode(q, Kc, Vc, o, kept, bits, tau, set(range(cfg.B * cfg.Hkv)))


def test_decode_group_sizes():
    rng = np.random.default_rng(3)
    for Hq, Hkv in ((4, 4), (8, 1), (16, 2)):
        B, Lc = 1, 3000
        q = dev_tensor(rng.standard_normal((B, Hq, 128)) * 2, torch.bfloat16)
        Kc = dev_tensor(rng.standard_normal((B, Hkv, Lc, 128)) * 2, torch.bfloat16)
        Vc = dev_tensor(rng.standard_normal((B, Hkv, Lc, 128)), torch.bfloat16)
        o, kept, bits = mala.mala_decode(q, Kc, Vc, tau=1.0, trace=True)
        mala.mala_check()
        check_decode(q, Kc, Vc, o, kept, bits, 1.0, set(range(B * Hkv)))


def test_empty_and_status():
    z = torch.empty((1, 1, 0, 128), dtype=torch.bfloat16, device="cuda")
    O, LSE = mala.mala_fwd(z, z, z)
    assert O.numel() == 0
    mala.mala_check()


@pytest.mark.parametrize("Lc,tau", [(5000, 1.0), (20000, 1.0), (3000, 4.0), (1000, 0.0)])
def test_decode_per_head_rows(Lc, tau):
    """Per-head rows: every query head applies the test alone (oracle flag
    per_head): keep sets per head, kept counts and outputs."""
    cfg = synth.DecodeConfig("per_head", 7, 2, 8, 2, Lc, 128, 128, 0.98, max(1, Lc // 256), 4)
    x = synth.decode_inputs(cfg)
    q = dev_tensor(x["q"], torch.bfloat16)
    Kc = dev_tensor(x["K"], torch.bfloat16)
    Vc = dev_tensor(x["V"], torch.bfloat16)
    o, kept, bits = mala.mala_decode(q, Kc, Vc, tau=tau, trace=True, per_head=True)
    mala.mala_check()
    nt = oracle.n_blocks(Lc, 128)
    B, Hq = q.shape[0], q.shape[1]
    gk = mala.unpack_bits(bits, nt)  # [B, Hq, nt]
    fewer = 0
    cov = Coverage(f"decode per-head rows Lc={Lc} tau={tau}")
    for b in range(B):
        ref = oracle.decode(rounded(q[b]), rounded(Kc[b]), rounded(Vc[b]), tau=tau, per_head=True,
                            want_margin=True)
        for h in range(Hq):
            cov.slices += 1
            if compare_decode_keep(gk[b, h], ref["keep"][h], ref["margin"][h]):
                cov.flips["decode"] += 1
                cov.add("o", np.zeros(1, bool))
                continue
            assert kept[b, h].item() == int(ref["keep"][h].sum())
            assert rel_l2(as_f64(o[b, h]), ref["o"][h]) <= TOL["bf16"]["decode"]
            cov.add("o", np.ones(1, bool))
            fewer += int(ref["keep"][h].sum())
    assert fewer > 0
    cov.require(0.75)


def gqa_case(L):
    """Two key/value heads of the matched_8k recipe, four query heads: query
    heads 0, 1 read kv head 0, heads 2, 3 read kv head 1 (each a copy of that
    head's own queries, the second one perturbed)."""
    cfg = synth.CONFIGS["matched_8k"]
    x = synth.prefill_inputs(cfg, L=L, heads=[0, 1])
    rng = np.random.default_rng(L + 17)
    Q = np.concatenate([x["Q"][:, :1], x["Q"][:, :1] + 0.3 * rng.standard_normal(x["Q"][:, :1].shape),
                        x["Q"][:, 1:2], 0.9 * x["Q"][:, 1:2]], axis=1)
    dO = rng.standard_normal(Q.shape)
    t = {"Q": dev_tensor(Q, torch.bfloat16), "dO": dev_tensor(dO, torch.bfloat16),
         "K": dev_tensor(x["K"][:, :2], torch.bfloat16), "V": dev_tensor(x["V"][:, :2], torch.bfloat16)}
    return t


@pytest.mark.parametrize("L,tau", [(1000, 1.0), (1536, 0.25), (640, 0.0)])
def test_bf16_grouped_query_heads(L, tau):
    """Grouped query heads (Hq = 4, Hkv = 2): per query head the rule on the
    shared K, V; dK, dV of a kv head are the sums over its query heads."""
    t = gqa_case(L)
    O, LSE, kept, bits, O32 = mala.mala_fwd(t["Q"], t["K"], t["V"], tau=tau, trace=True,
                                            o32=True)
    dQ, dK, dV, kept_b, bits_b = mala.mala_bwd(t["Q"], t["K"], t["V"], O, t["dO"], LSE, tau=tau,
                                               trace=True, o32=O32)
    mala.mala_check()
    nb = oracle.n_blocks(L, 128)
    Kd, Vd = [rounded(t["K"][0, g]) for g in range(2)], [rounded(t["V"][0, g]) for g in range(2)]
    refK, refV = [np.zeros_like(Kd[0]), np.zeros_like(Kd[0])], [np.zeros_like(Vd[0]), np.zeros_like(Vd[0])]
    kmasks = [np.ones(L, bool), np.ones(L, bool)]
    cov = Coverage(f"grouped heads L={L} tau={tau}")
    for h in range(4):
        g = h // 2
        Qd, dOd = rounded(t["Q"][0, h]), rounded(t["dO"][0, h])
        _, _, ref, bad = check_fwd_slice(Qd, Kd[g], Vd[g], as_f64(O[0, h]), as_f64(LSE[0, h]),
                                         bits[0, h], 128, tau, TOL["bf16"], cov=cov)
        gr = oracle.bwd(Qd, Kd[g], Vd[g], ref["O"], dOd, ref["LSE"], tile=128, tau=tau,
                        want_margin=True)
        gb = mala.unpack_bits(bits_b[0, h], nb)
        flips = compare_bwd_keep(gb, gr["keep"], gr["margin"], skip_blocks=bad)
        cov.flips["bwd"] += len(flips)
        qmask, kmask = grad_row_masks(L, 128, bad, flips, gb, gr["keep"])
        if qmask.any():
            assert rel_l2(as_f64(dQ[0, h])[qmask], gr["dQ"][qmask]) <= TOL["bf16"]["grad"]
        cov.add("dQ", qmask)
        kmasks[g] &= kmask  # a kv head's dK, dV sum over its query heads
        refK[g] += gr["dK"]
        refV[g] += gr["dV"]
    for g in range(2):
        m = kmasks[g]
        if m.any():
            assert rel_l2(as_f64(dK[0, g])[m], refK[g][m]) <= TOL["bf16"]["grad"]
            assert rel_l2(as_f64(dV[0, g])[m], refV[g][m]) <= TOL["bf16"]["grad"]
        cov.add("dK, dV", m)
    cov.require(0.5)


@pytest.mark.parametrize("tau", [1.0, 0.25])
def test_bf16_varlen_cache_append(tau):
    """Three packed sequences with (new queries, all keys) = (300, 300),
    (200, 500) (a cache of 300 keys: not a whole number of tiles) and
    (384, 640), two query heads on one key/value head: every (sequence,
    head) against the oracle's chunk forward (outputs, LSE, keep sets)."""
    lens = [(300, 300), (200, 500), (384, 640)]
    H, Hkv, d = 2, 1, 128
    rng = np.random.default_rng(91)
    cfg = synth.CONFIGS["matched_8k"]
    qs, ks, vs = [], [], []
    for s_i, (lq, lk) in enumerate(lens):
        x = synth.prefill_inputs(cfg, L=lk, heads=[s_i])
        K, V, Qall = x["K"][0, 0], x["V"][0, 0], x["Q"][0, 0]
        Qh = [Qall[lk - lq:], Qall[lk - lq:] * 0.8 + 0.2 * rng.standard_normal((lq, d))]
        qs.append(np.stack(Qh, axis=1))          # [lq, H, d]
        ks.append(K[:, None, :])
        vs.append(V[:, None, :])
    q = dev_tensor(np.concatenate(qs), torch.bfloat16)
    k = dev_tensor(np.concatenate(ks), torch.bfloat16)
    v = dev_tensor(np.concatenate(vs), torch.bfloat16)
    cq = torch.tensor(np.cumsum([0] + [a for a, _ in lens]), dtype=torch.int32).cuda()
    ck = torch.tensor(np.cumsum([0] + [b for _, b in lens]), dtype=torch.int32).cuda()
    mq, mk = max(a for a, _ in lens), max(b for _, b in lens)
    O, LSE, kept, bits = mala.mala_fwd_varlen(q, k, v, cq, ck, mq, mk, tau=tau, trace=True)
    mala.mala_check()
    cqh, ckh = cq.cpu().numpy(), ck.cpu().numpy()
    for b, (lq, lk) in enumerate(lens):
        Kd = rounded(k[ckh[b]:ckh[b + 1], 0])
        Vd = rounded(v[ckh[b]:ckh[b + 1], 0])
        for h in range(H):
            Qd = rounded(q[cqh[b]:cqh[b + 1], h])
            ref = oracle.fwd_chunk(Qd, Kd, Vd, tile=128, tau=tau, want_margin=True)
            nbq, nkt = ref["keep"].shape
            gk = mala.unpack_bits(bits[b, h], nkt)[:nbq]
            bad = []
            for i in range(nbq):
                diff = np.nonzero(gk[i] != ref["keep"][i])[0]
                if len(diff):
                    assert all(abs(ref["margin"][i, kk]) <= np.log1p(1e-3) for kk in diff), (b, h, i)
                    bad.append(i)
            rows = np.ones(lq, bool)
            for i in bad:  # a near-threshold flip changes that block's later tiles
                rows[i * 128:(i + 1) * 128] = False
            o = as_f64(O[cqh[b]:cqh[b + 1], h])
            assert rel_l2(o[rows], ref["O"][rows]) <= TOL["bf16"]["O"]
            assert rel_l2(as_f64(LSE[h, cqh[b]:cqh[b + 1]])[rows], ref["LSE"][rows]) <= TOL["bf16"]["LSE"]
            if not bad:
                assert np.array_equal(kept[b, h, :nbq].cpu().numpy(), ref["keep"].sum(axis=1))
