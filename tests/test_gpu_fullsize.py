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
from tests.parity import TOL, as_f64, compare_decode_keep, compare_fwd_keep, rel_l2

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
def prefill_run(inputs):
    P = bench.PREFILL
    shape = (P.B, P.H, P.L, P.d)
    t = {n: u16_to_dev(inputs["p" + n], shape) for n in ("Q", "K", "V", "dO")}
    O, LSE, kept, bits, O32, RM = mala.mala_fwd(t["Q"], t["K"], t["V"], tau=1.0, trace=True,
                                                o32=True, rowmax=True)
    dQ, dK, dV, kept_b, bits_b = mala.mala_bwd(t["Q"], t["K"], t["V"], O, t["dO"], LSE, tau=1.0,
                                               trace=True, o32=O32, rowmax=RM)
    del RM
    # the same test recomputing every tile's scores
    *_, kept_s, bits_s = mala.mala_bwd(t["Q"], t["K"], t["V"], O, t["dO"], LSE, tau=1.0,
                                       trace=True, o32=O32)
    mala.mala_check()
    same_test = torch.equal(bits_s, bits_b) and torch.equal(kept_s, kept_b)
    out = {"O": O, "LSE": LSE, "kept": kept, "bits": bits, "dQ": dQ, "dK": dK, "dV": dV,
           "kept_b": kept_b, "bits_b": bits_b, "same_test": same_test}
    del t
    return out


def head_f64(inputs, h):
    return {n: u16_to_f64(inputs["p" + n][h]) for n in ("Q", "K", "V", "dO")}


@pytest.mark.parametrize("h", [0, 5])
def test_long_128k_forward_sampled_blocks(inputs, prefill_run, h):
    L = bench.PREFILL.L
    nb = L // T
    x = head_f64(inputs, h)
    bits = mala.unpack_bits(prefill_run["bits"][0, h], nb)
    O = prefill_run["O"][0, h]
    LSE = prefill_run["LSE"][0, h]
    for lo, hi in ((0, 2), (511, 513), (nb - 3, nb)):
        ref = oracle.fwd(x["Q"], x["K"], x["V"], tile=T, tau=1.0, qblocks=(lo, hi), want_margin=True)
        _, bad = compare_fwd_keep(bits[lo:hi], ref["keep"][lo:hi], ref["margin"][lo:hi], lo)
        for i in range(lo, hi):
            if i - lo in bad:
                continue
            rows = slice(i * T, (i + 1) * T)
            assert rel_l2(as_f64(O[rows]), ref["O"][rows]) <= TOL["bf16"]["O"]
            assert rel_l2(as_f64(LSE[rows]), ref["LSE"][rows]) <= TOL["bf16"]["LSE"]


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
    assert prefill_run["same_test"]  # row-maxima test == recomputing test, bit for bit


def test_long_128k_backward_sampled_blocks(inputs, prefill_run):
    """dQ of the last query block and dK/dV of the last four key blocks of
    head 2 (their rows need only the last four query blocks' forward)."""
    h = 2
    L = bench.PREFILL.L
    nb = L // T
    x = head_f64(inputs, h)
    lo = nb - 4
    ref = oracle.fwd(x["Q"], x["K"], x["V"], tile=T, tau=1.0, qblocks=(lo, nb), want_margin=True)
    fbits = mala.unpack_bits(prefill_run["bits"][0, h], nb)
    _, bad = compare_fwd_keep(fbits[lo:nb], ref["keep"][lo:nb], ref["margin"][lo:nb], lo)
    assert not bad
    g = oracle.bwd(x["Q"], x["K"], x["V"], ref["O"], x["dO"], ref["LSE"], tile=T, tau=1.0,
                   qblocks=[nb - 1], kblocks=list(range(lo, nb)), want_margin=True)
    bbits = mala.unpack_bits(prefill_run["bits_b"][0, h], nb)
    # decisions the oracle visited: row nb-1 (every j), columns lo..nb-1
    visited = [(nb - 1, j) for j in range(nb)] + [(i, j) for j in range(lo, nb)
                                                    for i in range(j, nb)]
    for i, j in visited:
        if bbits[i, j] != g["keep"][i, j]:
            assert abs(g["margin"][i, j]) <= np.log1p(1e-3), (i, j)
    rows = slice((nb - 1) * T, nb * T)
    assert rel_l2(as_f64(prefill_run["dQ"][0, h][rows]), g["dQ"][rows]) <= TOL["bf16"]["grad"]
    krows = slice(lo * T, nb * T)
    for n in ("dK", "dV"):
        assert rel_l2(as_f64(prefill_run[n][0, h][krows]), g[n][krows]) <= TOL["bf16"]["grad"], n


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
    for flat in (0, 37, 77, 127):
        b, g = divmod(flat, Dc.Hkv)
        qs = q[b, g * G:(g + 1) * G]
        ref = oracle.decode(as_f64(qs), as_f64(Kc[b, g:g + 1]), as_f64(Vc[b, g:g + 1]), tau=1.0,
                            want_margin=True)
        if compare_decode_keep(allbits[b, g], ref["keep"][0], ref["margin"][0]):
            continue
        assert rel_l2(as_f64(o[b, g * G:(g + 1) * G]), ref["o"]) <= TOL["bf16"]["decode"]


@pytest.mark.parametrize("tau", [1.0, 0.0])
def test_sweep_32k_sampled(tau):
    cfg = synth.CONFIGS["sweep_L32768"]
    heads = [0, 11]
    x = synth.prefill_inputs(cfg, heads=heads)
    t = {n: torch.tensor(x[n]).to(torch.bfloat16).cuda() for n in ("Q", "K", "V")}
    O, LSE, kept, bits = mala.mala_fwd(t["Q"], t["K"], t["V"], tau=tau, trace=True)
    mala.mala_check()
    nb = cfg.L // T
    for h in heads:
        Qd, Kd, Vd = (as_f64(t[n][0, h]) for n in ("Q", "K", "V"))
        gbits = mala.unpack_bits(bits[0, h], nb)
        for lo, hi in ((100, 102), (nb - 2, nb)):
            ref = oracle.fwd(Qd, Kd, Vd, tile=T, tau=tau, qblocks=(lo, hi), want_margin=True)
            _, bad = compare_fwd_keep(gbits[lo:hi], ref["keep"][lo:hi], ref["margin"][lo:hi], lo)
            for i in range(lo, hi):
                if i - lo in bad:
                    continue
                rows = slice(i * T, (i + 1) * T)
                assert rel_l2(as_f64(O[0, h][rows]), ref["O"][rows]) <= TOL["bf16"]["O"]
                assert rel_l2(as_f64(LSE[0, h][rows]), ref["LSE"][rows]) <= TOL["bf16"]["LSE"]
