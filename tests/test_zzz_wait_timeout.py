"""Failure detection on the GPU without a fault: a device wait that runs out
(a barrier nothing arrives on, through the same bounded wait every kernel
uses) is reported once by mala_check as MALA_ERR_TIMEOUT, and the context
keeps computing correctly afterwards. Runs last: it holds one SM for the
wait's two seconds."""

import time

import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU container
    pytest.skip("needs a GPU", allow_module_level=True)

import mass_adaptive_causal_b200 as mala  # noqa: E402


def test_a_wait_that_runs_out_is_reported_once_and_the_context_stays_usable():
    torch.cuda.set_device(0)
    mala.mala_check()  # nothing pending before
    t0 = time.monotonic()
    mala.mala_selftest_wait()
    with pytest.raises(mala.MalaError, match="MALA_ERR_TIMEOUT"):
        mala.mala_check()
    waited = time.monotonic() - t0
    assert 1.5 < waited < 60  # the wait's limit, not a hang
    mala.mala_check()  # reported once, then cleared

    # the same context still computes: dense attention (tau = 0), its float32
    # output and LSE against causal softmax attention in float64 on the same
    # bf16 inputs
    g = torch.Generator().manual_seed(5)
    q, k, v = (torch.randn((1, 2, 384, 128), generator=g).to(torch.bfloat16).cuda()
               for _ in range(3))
    O, LSE, O32 = mala.mala_fwd(q, k, v, tau=0.0, o32=True)
    mala.mala_check()
    s = (q.double() @ k.double().transpose(-1, -2)) / 128 ** 0.5
    s = s.masked_fill(torch.triu(torch.ones(384, 384, dtype=torch.bool, device="cuda"), 1),
                      float("-inf"))
    ref = torch.softmax(s, dim=-1) @ v.double()
    assert ((O32.double() - ref).norm() / ref.norm()).item() <= 1e-3
    assert (LSE.double() - torch.logsumexp(s, dim=-1)).abs().max().item() <= 1e-3
