"""Matched-work study on the GPU path at the matched-work shape (L = 8192):
the keep set mala_fwd reports leaves out the same dense probability mass as
the oracle's keep set, up to the mass of tiles that flip inside the
near-threshold band, and at its own per-block budget it loses less mass than
a fixed position pattern and no less than the per-instance optimum
(MassAlloc Attention; jaehun.me review, "Matched-work study", Table 1)."""

from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth
from tests.parity import compare_fwd_keep

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU container
    pytest.skip("needs a GPU", allow_module_level=True)

import bench  # noqa: E402
import mass_adaptive_causal_b200 as mala  # noqa: E402

T = 128
HEADS = [0, 5]


def test_matched_8k_gpu_keep_set_omitted_mass():
    cfg = synth.CONFIGS["matched_8k"]
    L, d = cfg.L, cfg.d
    x = synth.prefill_inputs(cfg, heads=HEADS, with_grad=False)
    host = {n: bench.bf16_round(x[n][0, HEADS]) for n in ("Q", "K", "V")}  # (2, L, d)
    dev = {n: torch.from_numpy(host[n][None]).to(torch.bfloat16).cuda() for n in host}
    O, LSE, kept, bits = mala.mala_fwd(dev["Q"], dev["K"], dev["V"], tau=1.0, trace=True)
    mala.mala_check()
    nb = (L + T - 1) // T
    keep_gpu = mala.unpack_bits(bits, nb)[0]
    blk = np.arange(L) // T
    scale = 1.0 / np.sqrt(d)
    compared = 0
    for k in range(len(HEADS)):
        Q, K, V = host["Q"][k], host["K"][k], host["V"][k]
        f = oracle.fwd(Q, K, V, tile=T, tau=1.0, want_margin=True)
        compare_fwd_keep(keep_gpu[k], f["keep"], f["margin"])  # only near-threshold flips
        dense = oracle.dense_fwd(Q, K, V)
        om_ref = oracle.omitted_mass(Q, K, f["keep"], dense["LSE"], T)
        P, rm = bench.dense_row_tile_mass(Q, K, T, scale)
        # the host analysis agrees with the oracle on the oracle's keep set
        np.testing.assert_allclose(1.0 - (rm * f["keep"][blk]).sum(axis=1), om_ref, rtol=0,
                                   atol=1e-12)
        om_gpu = 1.0 - (rm * keep_gpu[k][blk]).sum(axis=1)
        flipped = (keep_gpu[k] != f["keep"]).astype(np.float64)
        allowance = (rm * flipped[blk]).sum(axis=1)
        assert np.all(np.abs(om_gpu - om_ref) <= allowance + 1e-12)
        # the same budget spent three ways
        counts = keep_gpu[k].sum(axis=1)
        om = {}
        for name, kp in (("mala", keep_gpu[k]), ("static", bench.position_static_keep(counts)),
                         ("oracle", bench.top_keep(bench.block_mass(rm, T), counts))):
            _, o = bench.restricted_output(P, V, kp, T)
            om[name] = o.mean()
        assert om["oracle"] <= om["mala"] + 1e-15
        assert om["mala"] < om["static"]
        compared += 1
    assert compared == len(HEADS)
