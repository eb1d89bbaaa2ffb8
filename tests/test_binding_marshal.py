"""The binding's entry points marshal their arguments as include/mala.h
declares them. A recording stand-in replaces the library's compute calls
(the size queries stay the real ones), the CUDA-only checks are relaxed so
that CPU tensors pass, and every entry point is called the way the GPU tests
and the benchmark call it."""

import ctypes

import pytest
import torch

import mass_adaptive_causal_b200 as mala

bf16, f32 = torch.bfloat16, torch.float32


class Recorder:
    COMPUTE = ("mala_fwd", "mala_fwd_varlen", "mala_bwd", "mala_decode", "mala_decode_noalloc",
               "mala_check", "mala_selftest_wait")

    def __init__(self, real):
        self.real = real
        self.calls = []

    def __getattr__(self, name):
        if name in self.COMPUTE:
            def call(*args):
                self.calls.append((name, args))
                return 0
            return call
        return getattr(self.real, name)


@pytest.fixture
def rec(monkeypatch):
    from mass_adaptive_causal_b200 import build
    build.build()
    r = Recorder(mala.lib())
    monkeypatch.setattr(mala, "_lib", r)
    real_inputs = mala._inputs
    monkeypatch.setattr(mala, "_inputs",
                        lambda ts, dev, require_cuda, what: real_inputs(ts, dev, False, what))
    monkeypatch.setattr(mala, "_stream", lambda stream: None)
    return r


def ptr(t):
    return t.data_ptr()


def val(a):
    return a.value if isinstance(a, ctypes.c_void_p) else a


def test_forward_and_backward(rec):
    B, H, Hkv, L, d = 1, 4, 2, 300, 128
    q = torch.randn((B, H, L, d)).to(bf16)
    k = torch.randn((B, Hkv, L, d)).to(bf16)
    v, do = torch.randn_like(k.float()).to(bf16), torch.randn_like(q.float()).to(bf16)
    O, LSE, kept, bits, O32 = mala.mala_fwd(q, k, v, tau=0.5, trace=True, o32=True)
    name, a = rec.calls[-1]
    assert name == "mala_fwd"
    a = [val(x) for x in a]
    assert a[0] == ptr(q) and a[1] == ptr(k) and a[2] == ptr(v) and a[3] == ptr(O)
    assert a[4] == ptr(LSE) and a[5] == ptr(O32)
    assert a[6:13] == [B, H, Hkv, L, d, mala.MALA_BF16, 0.5] and a[13] == 128
    assert a[15] == ptr(kept) and a[16] == ptr(bits)
    assert kept.shape == (B, H, 3) and bits.shape == (B, H, 3, 1)
    # the benchmark's form: every buffer passed in
    mala.mala_fwd(q, k, v, tau=1.0, out=O, lse=LSE, o32=O32)
    assert [val(x) for x in rec.calls[-1][1][3:6]] == [ptr(O), ptr(LSE), ptr(O32)]

    dQ, dK, dV, kb, bb = mala.mala_bwd(q, k, v, O, do, LSE, tau=0.5, trace=True, o32=O32)
    name, a = rec.calls[-1]
    a = [val(x) for x in a]
    assert name == "mala_bwd" and dK.shape == k.shape and dQ.shape == q.shape
    assert a[4] == ptr(O32) and a[5] == ptr(do) and a[6] == ptr(LSE)
    assert a[11] >= mala.bwd_workspace_bytes(B, H, L, d)
    assert a[12:19] == [B, H, Hkv, L, d, mala.MALA_BF16, 0.5]
    ws = torch.empty(mala.bwd_workspace_bytes(B, H, L, d), dtype=torch.uint8)
    grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(k))
    mala.mala_bwd(q, k, v, O, do, LSE, workspace=ws, grads=grads, o32=O32)
    a = [val(x) for x in rec.calls[-1][1]]
    assert a[7:12] == [ptr(grads[0]), ptr(grads[1]), ptr(grads[2]), ptr(ws), ws.numel()]
    mala.mala_check()
    assert rec.calls[-1][0] == "mala_check"


def test_float32_and_empty(rec):
    q = torch.randn((1, 1, 200, 64))
    O, LSE = mala.mala_fwd(q, q, q, tau=1.0)
    a = [val(x) for x in rec.calls[-1][1]]
    assert a[11] == mala.MALA_F32 and a[13] == 64 and O.dtype == f32
    z = torch.empty((1, 1, 0, 128), dtype=bf16)
    O, LSE = mala.mala_fwd(z, z, z)
    assert O.numel() == 0 and LSE.shape == (1, 1, 0)


def test_decode(rec):
    B, Hq, Hkv, Lc, d = 2, 8, 2, 1000, 128
    q = torch.zeros((B, Hq, d), dtype=bf16)
    kc = torch.zeros((B, Hkv, Lc, d), dtype=bf16)
    vc = torch.zeros_like(kc)
    o, kept, bits = mala.mala_decode(q, kc, vc, tau=1.0, trace=True, per_head=True)
    a = [val(x) for x in rec.calls[-1][1]]
    assert a[4:12] == [B, Hq, Hkv, Lc, d, 1.0, 0.0, 1]
    assert a[13] >= mala.decode_workspace_bytes(B, Hq, Hkv, Lc, d)
    assert kept.shape == (B, Hq) and bits.shape == (B, Hq, 1)
    ws = torch.empty(mala.decode_workspace_bytes(B, Hq, Hkv, Lc, d), dtype=torch.uint8)
    out = torch.empty_like(q)
    assert mala.mala_decode(q, kc, vc, workspace=ws, out=out) is out
    a = [val(x) for x in rec.calls[-1][1]]
    assert a[3] == ptr(out) and a[12] == ptr(ws) and a[13] == ws.numel()
    o, kept, bits = mala.mala_decode_noalloc(q, kc, vc, trace=True)
    name, a = rec.calls[-1]
    assert name == "mala_decode_noalloc" and kept.shape == (B, Hkv)
    assert [val(x) for x in a[4:9]] == [B, Hq, Hkv, Lc, d]


def test_varlen(rec):
    q = torch.zeros((150, 4, 128), dtype=bf16)
    k = torch.zeros((300, 2, 128), dtype=bf16)
    cq = torch.tensor([0, 100, 150], dtype=torch.int32)
    ck = torch.tensor([0, 200, 300], dtype=torch.int32)
    O, LSE, kept, bits = mala.mala_fwd_varlen(q, k, k, cq, ck, 100, 200, tau=1.0, trace=True)
    a = [val(x) for x in rec.calls[-1][1]]
    assert a[5] == ptr(cq) and a[6] == ptr(ck)
    assert a[7:15] == [2, 100, 200, 150, 300, 4, 2, 128]
    assert LSE.shape == (4, 150) and kept.shape == (2, 4, 1)
    assert bits.shape == (2, 4, 1, mala.lib().mala_varlen_trace_words(100, 200))


def test_selftest_wait(rec):
    mala.mala_selftest_wait()
    assert rec.calls[-1][0] == "mala_selftest_wait"
