"""GPU parity at the benchmark's full sizes, in the launch configuration the
benchmark times, on sampled outputs the oracle can compute block by block,
plus properties that hold at any size.

long_128k: B=1 H=8 L=131072 d=128 bf16 tile 128, tau=1 (forward, backward);
decode_128k: B=16 Hq=32 Hkv=8 Lc=131072 d=128 bf16, tau=1;
sweep_L32768: B=1 H=16 L=32768 d=128 bf16, tau=1 and tau=0.
"""

from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth
from tests.parity import (TOL, Coverage, as_f64, compare_bwd_keep, compare_decode_keep,
                          compare_fwd_keep, grad_row_masks, rel_l2)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU container
    pytest.skip("needs a GPU", allow_module_level=True)

import bench  # noqa: E402  (input generation shared with the benchmark)
import mass_adaptive_causal_b200 as mala  # noqa: E402

T = 128


@pytest.fixture(scope="module")
def inputs():
    """The benchmark's inputs (uint16 bf16 bit patterns), generated with a
    spawn pool exactly as bench.py does."""
    return bench.generate_inputs(workers=16)


def u16_to_dev(u16, shape):
    return torch.from_numpy(u16.view(np.int16)).view(torch.bfloat16).reshape(shape).cuda()


def u16_to_f64(u16):
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.fixture(scope="module")
def prefill_dev(inputs):
    P = bench.PREFILL
    shape = (P.B, P.H, P.L, P.d)
    return {n: u16_to_dev(inputs["p" + n], shape) for n in ("Q", "K", "V", "dO")}


@pytest.fixture(scope="module")
def prefill_run(prefill_dev):
    """The benchmark's training chain at tau=1: forward, then the backward
    from O (float32 copy) and LSE only."""
    t = prefill_dev
    O, LSE, kept, bits, O32 = mala.mala_fwd(t["Q"], t["K"], t["V"], tau=1.0, trace=True, o32=True)
    dQ, dK, dV, kept_b, bits_b = mala.mala_bwd(t["Q"], t["K"], t["V"], O, t["dO"], LSE, tau=1.0,
                                               trace=True, o32=O32)
    mala.mala_check()
    return {"O": O, "LSE": LSE, "kept": kept, "bits": bits, "dQ": dQ, "dK": dK, "dV": dV,
            "kept_b": kept_b, "bits_b": bits_b}


def head_f64(inputs, h):
    return {n: u16_to_f64(inputs["p" + n][h]) for n in ("Q", "K", "V", "dO")}


def check_fwd_blocks(x, O, LSE, gbits, tau, ranges, cov):
    """Forward rows of the query-block ranges against the oracle run on those
    blocks only."""
    for lo, hi in ranges:
        ref = oracle.fwd(x["Q"], x["K"], x["V"], tile=T, tau=tau, qblocks=(lo, hi),
                         want_margin=True)
        n_near, bad = compare_fwd_keep(gbits[lo:hi], ref["keep"][lo:hi], ref["margin"][lo:hi], lo)
        cov.flips["fwd"] += n_near
        for i in range(lo, hi):
            ok = (i - lo) not in bad
            cov.add("O", np.full(T, ok))
            if not ok:
                continue
            rows = slice(i * T, (i + 1) * T)
            assert rel_l2(as_f64(O[rows]), ref["O"][rows]) <= TOL["bf16"]["O"]
            assert rel_l2(as_f64(LSE[rows]), ref["LSE"][rows]) <= TOL["bf16"]["LSE"]


def check_bwd_tail(x, fbits, bbits, dQ, dK, dV, tau, nb, cov, nk=4):
    """dQ of the last query block and dK, dV of the last ``nk`` key blocks of
    one head (their rows need only the last ``nk`` query blocks' forward).
    The oracle's backward is fed the oracle's own forward of those blocks."""
    lo = nb - nk
    ref = oracle.fwd(x["Q"], x["K"], x["V"], tile=T, tau=tau, qblocks=(lo, nb), want_margin=True)
    n_near, bad = compare_fwd_keep(fbits[lo:nb], ref["keep"][lo:nb], ref["margin"][lo:nb], lo)
    cov.flips["fwd"] += n_near
    bad = [b + lo for b in bad]
    g = oracle.bwd(x["Q"], x["K"], x["V"], np.nan_to_num(ref["O"]), x["dO"],
                   np.nan_to_num(ref["LSE"]), tile=T, tau=tau, qblocks=[nb - 1],
                   kblocks=list(range(lo, nb)), want_margin=True)
    # the decisions the oracle visited: row nb - 1 (every j), columns lo..nb-1
    visited = np.zeros((nb, nb), bool)
    visited[nb - 1, :] = True
    for j in range(lo, nb):
        visited[j:, j] = True
    visited &= np.tril(np.ones((nb, nb), bool))
    gk = np.where(visited, bbits, 0)
    rk = np.where(visited, g["keep"], 0)
    flips = compare_bwd_keep(gk, rk, g["margin"], skip_blocks=bad)
    cov.flips["bwd"] += len(flips)
    L = nb * T
    qmask, kmask = grad_row_masks(L, T, bad, flips, gk, rk)
    qrows = np.zeros(L, bool)
    qrows[(nb - 1) * T:] = True
    krows = np.zeros(L, bool)
    krows[lo * T:] = True
    qm, km = qmask & qrows, kmask & krows
    if qm.any():
        assert rel_l2(as_f64(dQ)[qm], g["dQ"][qm]) <= TOL["bf16"]["grad"]
    for n, a in (("dK", dK), ("dV", dV)):
        if km.any():
            assert rel_l2(as_f64(a)[km], g[n][km]) <= TOL["bf16"]["grad"], n
    cov.add("dQ", qm[qrows])
    cov.add("dK, dV", km[krows])


@pytest.mark.parametrize("h", [0, 5])
def test_long_128k_forward_sampled_blocks(inputs, prefill_run, h):
    nb = bench.PREFILL.L // T
    cov = Coverage(f"long_128k forward head {h}")
    check_fwd_blocks(head_f64(inputs, h), prefill_run["O"][0, h], prefill_run["LSE"][0, h],
                     mala.unpack_bits(prefill_run["bits"][0, h], nb), 1.0,
                     ((0, 2), (511, 513), (nb - 3, nb)), cov)
    cov.require(0.5)


def test_long_128k_dense_forward_sampled_blocks(inputs, prefill_dev):
    """tau = 0 (the in-house dense comparison) at the benchmark's size: every
    tile kept, outputs of sampled blocks of head 3 equal dense attention's."""
    t = prefill_dev
    O, LSE, kept, bits = mala.mala_fwd(t["Q"], t["K"], t["V"], tau=0.0, trace=True)
    mala.mala_check()
    nb = bench.PREFILL.L // T
    assert np.array_equal(kept[0].cpu().numpy(), np.tile(np.arange(1, nb + 1), (bench.PREFILL.H, 1)))
    h = 3
    cov = Coverage("long_128k dense forward head 3")
    check_fwd_blocks(head_f64(inputs, h), O[0, h], LSE[0, h], mala.unpack_bits(bits[0, h], nb),
                     0.0, ((0, 1), (700, 701), (nb - 2, nb)), cov)
    cov.require(1.0)


def test_long_128k_keep_properties(prefill_run):
    """At any size: every query block keeps its diagonal; kept_tiles equals the
    popcount of each keep-bit row (forward) / column (backward); nothing above
    the diagonal; backward keeps fewer tiles than forward overall."""
    nb = bench.PREFILL.L // T
    for h in range(bench.PREFILL.H):
        f = mala.unpack_bits(prefill_run["bits"][0, h], nb)
        b = mala.unpack_bits(prefill_run["bits_b"][0, h], nb)
        assert np.all(np.diag(f) == 1)
        assert not np.any(np.triu(f, 1)) and not np.any(np.triu(b, 1))
        assert np.array_equal(prefill_run["kept"][0, h].cpu().numpy(), f.sum(axis=1))
        assert np.array_equal(prefill_run["kept_b"][0, h].cpu().numpy(), b.sum(axis=0))
        assert b.sum() <= f.sum()


@pytest.mark.parametrize("h", [2, 4, 7])
def test_long_128k_backward_sampled_blocks(inputs, prefill_run, h):
    """dQ of the last query block and dK/dV of the last four key blocks."""
    nb = bench.PREFILL.L // T
    cov = Coverage(f"long_128k backward head {h}")
    check_bwd_tail(head_f64(inputs, h), mala.unpack_bits(prefill_run["bits"][0, h], nb),
                   mala.unpack_bits(prefill_run["bits_b"][0, h], nb), prefill_run["dQ"][0, h],
                   prefill_run["dK"][0, h], prefill_run["dV"][0, h], 1.0, nb, cov)
    cov.require(0.5)


def test_decode_128k_sampled_groups(inputs):
    Dc = bench.DECODE
    G = Dc.Hq // Dc.Hkv
    q = u16_to_dev(inputs["dq"], (Dc.B, Dc.Hq, Dc.d))
    Kc = u16_to_dev(inputs["dK"], (Dc.B, Dc.Hkv, Dc.Lc, Dc.d))
    Vc = u16_to_dev(inputs["dV"], (Dc.B, Dc.Hkv, Dc.Lc, Dc.d))
    o, kept, bits = mala.mala_decode(q, Kc, Vc, tau=1.0, trace=True)
    mala.mala_check()
    nt = Dc.Lc // T
    allbits = mala.unpack_bits(bits, nt)
    assert np.array_equal(kept.cpu().numpy(), allbits.sum(axis=-1))
    assert np.all(allbits[..., nt - 1] == 1)  # newest tile always kept
    cov = Coverage("decode_128k sampled groups")
    for flat in (0, 13, 37, 50, 77, 90, 111, 127):
        b, g = divmod(flat, Dc.Hkv)
        qs = q[b, g * G:(g + 1) * G]
        ref = oracle.decode(as_f64(qs), as_f64(Kc[b, g:g + 1]), as_f64(Vc[b, g:g + 1]), tau=1.0,
                            want_margin=True)
        cov.slices += 1
        if compare_decode_keep(allbits[b, g], ref["keep"][0], ref["margin"][0]):
            cov.flips["decode"] += 1
            cov.add("o", np.zeros(1, bool))
            continue
        assert kept[b, g].item() == int(ref["keep"][0].sum())
        assert rel_l2(as_f64(o[b, g * G:(g + 1) * G]), ref["o"]) <= TOL["bf16"]["decode"]
        cov.add("o", np.ones(1, bool))
    cov.require(0.75)


@pytest.mark.parametrize("tau", [1.0, 0.0])
def test_sweep_32k_sampled(tau):
    """sweep_L32768 (H=16), heads 0 and 11: forward rows of sampled query
    blocks, and the backward's dQ of the last query block and dK, dV of the
    last four key blocks."""
    cfg = synth.CONFIGS["sweep_L32768"]
    heads = [0, 11]
    x = synth.prefill_inputs(cfg, heads=heads)
    t = {n: torch.tensor(x[n]).to(torch.bfloat16).cuda() for n in ("Q", "K", "V", "dO")}
    O, LSE, kept, bits, O32 = mala.mala_fwd(t["Q"], t["K"], t["V"], tau=tau, trace=True, o32=True)
    dQ, dK, dV, kept_b, bits_b = mala.mala_bwd(t["Q"], t["K"], t["V"], O, t["dO"], LSE, tau=tau,
                                               trace=True, o32=O32)
    mala.mala_check()
    nb = cfg.L // T
    fcov = Coverage(f"sweep_L32768 forward tau={tau}")
    bcov = Coverage(f"sweep_L32768 backward tau={tau}")
    for k in range(len(heads)):
        xd = {n: as_f64(t[n][0, k]) for n in ("Q", "K", "V", "dO")}
        fb = mala.unpack_bits(bits[0, k], nb)
        check_fwd_blocks(xd, O[0, k], LSE[0, k], fb, tau, ((100, 102), (nb - 2, nb)), fcov)
        check_bwd_tail(xd, fb, mala.unpack_bits(bits_b[0, k], nb), dQ[0, k], dK[0, k], dV[0, k],
                       tau, nb, bcov)
    fcov.require(0.5)
    bcov.require(0.5)
