"""How the backward's bf16 operands of dS bound the gradients' error.

The work pass multiplies dS = P o (dP - D) * scale by Q (for dK) and by K (for
dQ) on the tensor cores, so dS must be rounded to bf16 first. dQ_r sums
dS_rc K_c over keys c, and every full row of dS sums to zero, so dQ is a
cancelling sum: one bf16 rounding of dS costs it most of the 1e-2 gradient
tolerance, and the kernel feeds the dQ product a pair hi + lo (~16 bits).
dK_c sums dS_rc Q_r over queries r, where dS has no such structure, so the
kernel gives the dK product hi alone. These checks hold that reasoning to the
synthetic recipes: dense causal attention at L = 1024 (every key kept), in
float64 apart from the rounding under test (round to nearest even, as the
kernel's conversion)."""

from __future__ import annotations

import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")

L = 1024
RECIPES = ["sweep_L1024", "long_128k", "matched_8k"]


def _bf16(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(a).to(torch.bfloat16).to(torch.float64).numpy()


def _rel(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("recipe", RECIPES)
def test_single_bf16_ds_suffices_for_dk_not_for_dq(recipe):
    x = synth.prefill_inputs(synth.CONFIGS[recipe], L=L, heads=[0])
    Q, K, V = (_bf16(np.asarray(x[n][0, 0], dtype=np.float64)) for n in ("Q", "K", "V"))
    dO = _bf16(np.random.default_rng(7).standard_normal(Q.shape) * 0.1)
    scale = 1.0 / np.sqrt(Q.shape[1])
    S = np.where(np.tril(np.ones((L, L), dtype=bool)), Q @ K.T * scale, -np.inf)
    P = np.exp(S - S.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    D = (dO * (P @ V)).sum(axis=1)
    dS = P * (dO @ V.T - D[:, None]) * scale
    # each full row of dS sums to zero: the cancellation dQ inherits
    np.testing.assert_allclose(dS.sum(axis=1), 0.0, atol=1e-12)
    dK, dQ = dS.T @ Q, dS @ K
    hi = _bf16(dS)
    lo = _bf16(dS - hi)
    err_dk = _rel(hi.T @ Q, dK)
    err_dq_hi = _rel(hi @ K, dQ)
    err_dq_pair = _rel((hi + lo) @ K, dQ)
    assert err_dk < 3e-3            # dK: hi alone, a small part of the 1e-2 tolerance
    assert err_dq_hi > 5e-3         # dQ: hi alone would spend most of it
    assert err_dq_pair < 1e-4       # dQ: the pair leaves it at float32-like accuracy
    assert err_dq_hi > 3 * err_dk
