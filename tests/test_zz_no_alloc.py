"""mala_decode_noalloc (the decode step whose scratch is the library's static
device array) against mala_decode (caller-provided workspace), through the C
ABI, on two calls in a row with different shapes, so that the second call
runs over the first call's leftovers in the shared array. The file sorts
after the parity tests so that it runs after them as well as alone."""

from __future__ import annotations

import pytest

import synth
from tests.parity import TOL, as_f64, rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU container
    pytest.skip("needs a GPU", allow_module_level=True)

import mass_adaptive_causal_b200 as mala  # noqa: E402


def _inputs(cfg):
    x = synth.decode_inputs(cfg)
    return tuple(torch.tensor(x[n]).to(torch.bfloat16).cuda() for n in ("q", "K", "V"))


CASES = [
    # (config, tau): the first call leaves 8 groups x 157 tiles of statistics
    # and lists behind; the second has fewer groups and a shorter cache.
    (synth.DecodeConfig("noalloc_a", 11, 2, 16, 4, 20000, 128, 128, 0.98, 40, 4), 1.0),
    (synth.DecodeConfig("noalloc_b", 12, 2, 8, 2, 5000, 128, 128, 0.98, 10, 4), 0.5),
]


def test_noalloc_decode_matches_workspace_decode_on_two_calls():
    for cfg, tau in CASES:
        q, Kc, Vc = _inputs(cfg)
        need = mala.decode_workspace_bytes(cfg.B, cfg.Hq, cfg.Hkv, cfg.Lc, cfg.d)
        assert need <= mala.NOALLOC_SCRATCH_BYTES
        o_ref, kept_ref, bits_ref = mala.mala_decode(q, Kc, Vc, tau=tau, trace=True)
        mala.mala_check()
        o, kept, bits = mala.mala_decode_noalloc(q, Kc, Vc, tau=tau, trace=True)
        mala.mala_check()
        assert torch.equal(kept, kept_ref)
        assert torch.equal(bits, bits_ref)
        assert rel_l2(as_f64(o), as_f64(o_ref)) <= TOL["bf16"]["decode"]
        assert torch.isfinite(o.float()).all()


def test_noalloc_decode_rejects_shapes_beyond_the_scratch():
    # statistics alone: 64 x 64 heads x 256 tiles x 8 bytes = 8 MiB + the rest.
    # The buffers have the declared sizes (4 GiB per cache), so nothing
    # would be read out of bounds even if the check let the call through.
    B, Hq, Hkv, Lc, d = 64, 64, 8, 32768, 128
    assert mala.decode_workspace_bytes(B, Hq, Hkv, Lc, d) > mala.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((B, Hq, d), dtype=torch.bfloat16, device="cuda")
    Kc = torch.zeros((B, Hkv, Lc, d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mala.MalaError, match="MALA_ERR_TOO_LARGE"):
        mala.mala_decode_noalloc(q, Kc, Kc, tau=1.0)
    del Kc
    torch.cuda.empty_cache()
