"""The binding's host checks, on CPU tensors: the C ABI gets bare pointers,
so every shape, dtype, byte count and device it relies on is checked in
Python before the call. The happy paths here are the shapes the GPU tests
and the benchmark pass."""

import pytest
import torch

import mass_adaptive_causal_b200 as mala

bf16, f32 = torch.bfloat16, torch.float32


@pytest.fixture(scope="module", autouse=True)
def built():
    from mass_adaptive_causal_b200 import build
    build.build()


def prefill(B=2, H=4, Hkv=2, L=300, d=128, dtype=bf16):
    q = torch.zeros((B, H, L, d), dtype=dtype)
    k = torch.zeros((B, Hkv, L, d), dtype=dtype)
    return q, k, torch.zeros_like(k)


def test_prefill_inputs():
    q, k, v = prefill()
    mala._check_prefill(q, k, v, q.clone(), q.clone(), require_cuda=False)
    with pytest.raises(ValueError, match="CUDA"):
        mala._check_prefill(q, k, v)
    with pytest.raises(ValueError, match="contiguous"):
        mala._check_prefill(q.transpose(2, 3), k, v, require_cuda=False)
    with pytest.raises(ValueError, match="one device"):
        mala._check_prefill(q, k.to("meta"), v, require_cuda=False)
    with pytest.raises(ValueError, match="one dtype"):
        mala._check_prefill(q, k.float(), v, require_cuda=False)
    with pytest.raises(ValueError, match="K and V"):
        mala._check_prefill(q, k, v[:, :, :10].contiguous(), require_cuda=False)
    q3, k3, v3 = prefill(H=4, Hkv=3)
    with pytest.raises(ValueError, match="multiple"):
        mala._check_prefill(q3, k3, v3, require_cuda=False)
    with pytest.raises(ValueError, match="Q's shape"):
        mala._check_prefill(q, k, v, q[:1].contiguous(), require_cuda=False)


def test_forward_buffers():
    q, _, _ = prefill()
    B, H, L, _ = q.shape
    good = dict(out=torch.empty_like(q), lse=torch.empty((B, H, L), dtype=f32),
                o32=torch.empty(q.shape, dtype=f32))
    mala._check_fwd_buffers(q, **good)
    mala._check_fwd_buffers(q)
    for name, bad, msg in (
            ("out", torch.empty((B, H, L - 1, 128), dtype=bf16), "shape"),
            ("out", torch.empty(q.shape, dtype=f32), "must be"),
            ("lse", torch.empty((B, H, L), dtype=bf16), "must be"),
            ("lse", torch.empty((B * H * L,), dtype=f32), "shape"),
            ("o32", torch.empty(q.shape, dtype=bf16), "must be"),
            ("out", torch.empty(q.shape, dtype=bf16, device="meta"), "must be on")):
        with pytest.raises(ValueError, match=msg):
            mala._check_fwd_buffers(q, **dict(good, **{name: bad}))


def test_backward_buffers():
    q, k, _ = prefill()
    B, H, L, _ = q.shape
    lse = torch.empty((B, H, L), dtype=f32)
    grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(k))
    ws = torch.empty(mala.bwd_workspace_bytes(B, H, L, 128), dtype=torch.uint8)
    mala._check_bwd_buffers(q, k, lse, o32=torch.empty(q.shape, dtype=f32), grads=grads,
                            workspace=ws)
    mala._check_bwd_buffers(q, k, lse)
    with pytest.raises(ValueError, match="lse"):
        mala._check_bwd_buffers(q, k, lse[:, :1].contiguous())
    with pytest.raises(ValueError, match="o32"):
        mala._check_bwd_buffers(q, k, lse, o32=torch.empty(q.shape, dtype=bf16))
    with pytest.raises(ValueError, match="dK"):  # grouped heads: dK has K's shape
        mala._check_bwd_buffers(q, k, lse, grads=(grads[0], torch.empty_like(q), grads[2]))
    with pytest.raises(ValueError, match="workspace"):
        mala._check_bwd_buffers(q, k, lse, workspace=torch.empty((64, 64))[:, ::2])


def decode(B=2, Hq=8, Hkv=2, Lc=1000, d=128):
    return (torch.zeros((B, Hq, d), dtype=bf16), torch.zeros((B, Hkv, Lc, d), dtype=bf16),
            torch.zeros((B, Hkv, Lc, d), dtype=bf16))


def test_decode_inputs():
    q, kc, vc = decode()
    ws = torch.empty(mala.decode_workspace_bytes(2, 8, 2, 1000, 128), dtype=torch.uint8)
    mala._check_decode(q, kc, vc, out=torch.empty_like(q), workspace=ws, require_cuda=False)
    mala._check_decode(q, kc, kc, require_cuda=False)  # one tensor as both caches
    with pytest.raises(ValueError, match="CUDA"):
        mala._check_decode(q, kc, vc)
    with pytest.raises(ValueError, match="one shape"):
        mala._check_decode(q, kc, vc[:, :, :500].contiguous(), require_cuda=False)
    with pytest.raises(ValueError, match="one shape"):
        mala._check_decode(q[None], kc, vc, require_cuda=False)
    with pytest.raises(ValueError, match="B and d"):
        mala._check_decode(q[:1].contiguous(), kc, vc, require_cuda=False)
    with pytest.raises(ValueError, match="B and d"):
        mala._check_decode(q[..., :64].contiguous(), kc, vc, require_cuda=False)
    with pytest.raises(ValueError, match="bf16"):
        mala._check_decode(q.float(), kc, vc, require_cuda=False)
    with pytest.raises(ValueError, match="out"):
        mala._check_decode(q, kc, vc, out=torch.empty((2, 8, 64), dtype=bf16),
                           require_cuda=False)


def test_varlen_inputs():
    q = torch.zeros((150, 4, 128), dtype=bf16)
    k = torch.zeros((300, 2, 128), dtype=bf16)
    cq = torch.tensor([0, 100, 150], dtype=torch.int32)
    ck = torch.tensor([0, 200, 300], dtype=torch.int32)
    mala._check_varlen(q, k, k.clone(), cq, ck, out=torch.empty_like(q),
                       lse=torch.empty((4, 150), dtype=f32), require_cuda=False)
    with pytest.raises(ValueError, match="CUDA"):
        mala._check_varlen(q, k, k, cq, ck)
    with pytest.raises(ValueError, match="one shape"):
        mala._check_varlen(q, k, k[:10].contiguous(), cq, ck, require_cuda=False)
    with pytest.raises(ValueError, match="int32"):
        mala._check_varlen(q, k, k, cq.long(), ck, require_cuda=False)
    with pytest.raises(ValueError, match="batch"):
        mala._check_varlen(q, k, k, cq, ck[:2].contiguous(), require_cuda=False)
    with pytest.raises(ValueError, match="batch"):
        mala._check_varlen(q, k, k, cq[:1].contiguous(), ck[:1].contiguous(),
                           require_cuda=False)
    with pytest.raises(ValueError, match="lse"):
        mala._check_varlen(q, k, k, cq, ck, lse=torch.empty((150, 4), dtype=f32),
                           require_cuda=False)
