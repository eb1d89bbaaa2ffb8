"""MALA (MassAlloc Attention) for NVIDIA B200 -- Python binding of the C ABI.

This module only marshals arguments: torch tensors supply device memory and
the current CUDA stream; every step of the computation runs in the kernels of
``libmala.so`` (built from ``csrc/`` for sm_100a). There is no fallback: if
the library is missing or fails to load, every call raises.

Entry points (same names as the C ABI in ``include/mala.h``):

* :func:`mala_fwd`    -- forward / prefill: O, LSE
* :func:`mala_bwd`    -- backward: dQ, dK, dV
* :func:`mala_decode` -- one decode step over a KV cache: o
* :func:`mala_check`  -- synchronize and read the device status word
"""

from __future__ import annotations

import ctypes
import os

__all__ = ["mala_fwd", "mala_fwd_varlen", "mala_bwd", "mala_decode", "mala_decode_noalloc", "mala_check",
           "mala_selftest_wait", "MalaError", "lib",
           "LIB_PATH", "MALA_F32", "MALA_BF16", "STATUS"]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmala.so")

MALA_F32, MALA_BF16 = 0, 1
STATUS = {0: "MALA_OK", 1: "MALA_ERR_INVALID_ARG", 2: "MALA_ERR_UNSUPPORTED",
          3: "MALA_ERR_CUDA", 4: "MALA_ERR_TIMEOUT", 5: "MALA_ERR_TOO_LARGE"}


class MalaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


_lib = None
_vp, _i32p, _u32p, _fp = (ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p)


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m mass_adaptive_causal_b200.build`"
                " (or __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        ci, cf, cs = ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.mala_fwd.argtypes = [_vp, _vp, _vp, _vp, _fp, _fp, ci, ci, ci, ci, ci, ci, cf, ci, cf,
                               _i32p, _u32p, _vp]
        L.mala_fwd_varlen.argtypes = [_vp, _vp, _vp, _vp, _fp, _vp, _vp, ci, ci, ci, ci, ci, ci,
                                      ci, ci, cf, ci, cf, _i32p, _u32p, _vp]
        L.mala_fwd_varlen.restype = ci
        L.mala_varlen_trace_words.argtypes = [ci, ci]
        L.mala_varlen_trace_words.restype = ci
        L.mala_fwd.restype = ci
        L.mala_bwd_workspace_bytes.argtypes = [ci, ci, ci, ci]
        L.mala_bwd_workspace_bytes.restype = cs
        L.mala_bwd.argtypes = [_vp, _vp, _vp, _vp, _fp, _vp, _fp, _vp, _vp, _vp, _vp, cs, ci, ci,
                               ci, ci, ci, ci, cf, ci, cf, _i32p, _u32p, _vp]
        L.mala_bwd.restype = ci
        L.mala_decode_workspace_bytes.argtypes = [ci, ci, ci, ci, ci]
        L.mala_decode_workspace_bytes.restype = cs
        L.mala_decode.argtypes = [_vp, _vp, _vp, _vp, ci, ci, ci, ci, ci, cf, cf, ci, _vp, cs,
                                  _i32p, _u32p, _vp]
        L.mala_decode.restype = ci
        L.mala_decode_noalloc.argtypes = [_vp, _vp, _vp, _vp, ci, ci, ci, ci, ci, cf, cf, _i32p,
                                          _u32p, _vp]
        L.mala_decode_noalloc.restype = ci
        L.mala_check.argtypes = [_vp]
        L.mala_check.restype = ci
        L.mala_selftest_wait.argtypes = [_vp]
        L.mala_selftest_wait.restype = ci
        L.mala_status_string.argtypes = [ci]
        L.mala_status_string.restype = ctypes.c_char_p
        L.mala_version.argtypes = []
        L.mala_version.restype = ci
        _lib = L
    return _lib


def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.float32:
        return MALA_F32
    if t.dtype == torch.bfloat16:
        return MALA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


# ---------------------------------------------------------------------------
# host checks: the C ABI receives bare pointers, so every size it relies on
# is checked here against the tensors before a pointer crosses. Each check
# takes ``require_cuda`` so that its logic runs on CPU tensors in the tests.
# ---------------------------------------------------------------------------
def _inputs(ts, dev, require_cuda, what):
    for t in ts:
        if require_cuda and not t.is_cuda:
            raise ValueError(f"{what} must be CUDA tensors")
        if not t.is_contiguous():
            raise ValueError(f"{what} must be contiguous")
        if t.device != dev:
            raise ValueError("every tensor of a call must be on one device")
    if require_cuda and dev.index != _torch().cuda.current_device():
        raise ValueError(f"the tensors are on {dev}, not on the current CUDA device "
                         "(torch.cuda.set_device)")


def _buf(t, name, dev, dtype, shape=None, min_bytes=None):
    """A caller-supplied output or scratch tensor: contiguous, on ``dev``, of
    ``dtype`` (any when None), exactly ``shape`` and/or at least ``min_bytes``."""
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device != dev:
        raise ValueError(f"{name} must be on {dev}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if min_bytes is not None and t.numel() * t.element_size() < min_bytes:
        raise ValueError(f"{name} holds {t.numel() * t.element_size()} bytes, needs {min_bytes}")
    return t


def _check_prefill(q, k, v, *rest, require_cuda=True):
    """q (and o, do in rest): [B, H, L, d]; k, v: [B, Hkv, L, d] with H % Hkv == 0
    (grouped query heads; Hkv = H is multi-head attention)."""
    torch = _torch()
    _inputs((q, k, v) + rest, q.device, require_cuda, "Q, K, V, O, dO")
    for t in (q, k, v) + rest:
        if t.dtype != q.dtype or t.dim() != 4:
            raise ValueError("expected [B, H, L, d] tensors of one dtype")
    if k.shape != v.shape or k.shape[0] != q.shape[0] or k.shape[2:] != q.shape[2:]:
        raise ValueError("K and V must be [B, Hkv, L, d] matching Q's B, L, d")
    if k.shape[1] == 0 or q.shape[1] % k.shape[1] != 0:
        raise ValueError("the query heads must be a multiple of the key/value heads")
    for t in rest:
        if t.shape != q.shape:
            raise ValueError("O and dO must have Q's shape")
    return torch


def _check_fwd_buffers(q, out=None, lse=None, o32=None):
    torch = _torch()
    B, H, L, _ = q.shape
    if out is not None:
        _buf(out, "out", q.device, q.dtype, q.shape)
    if lse is not None:
        _buf(lse, "lse", q.device, torch.float32, (B, H, L))
    if o32 is not None:
        _buf(o32, "o32", q.device, torch.float32, q.shape)


def _check_bwd_buffers(q, k, lse, o32=None, grads=None, workspace=None):
    torch = _torch()
    B, H, L, _ = q.shape
    _buf(lse, "lse", q.device, torch.float32, (B, H, L))
    if o32 is not None:
        _buf(o32, "o32", q.device, torch.float32, q.shape)
    if grads is not None:
        dq, dk, dv = grads
        _buf(dq, "dQ", q.device, q.dtype, q.shape)
        _buf(dk, "dK", q.device, q.dtype, k.shape)
        _buf(dv, "dV", q.device, q.dtype, k.shape)
    if workspace is not None:
        _buf(workspace, "workspace", q.device, None)


def _check_decode(q, k_cache, v_cache, out=None, workspace=None, require_cuda=True):
    """q: [B, Hq, d] bf16; caches: [B, Hkv, Lc, d] bf16, the same shape."""
    torch = _torch()
    _inputs((q, k_cache, v_cache), q.device, require_cuda, "decode tensors")
    for t in (q, k_cache, v_cache):
        if t.dtype != torch.bfloat16:
            raise ValueError("decode tensors must be bf16")
    if q.dim() != 3 or k_cache.dim() != 4 or k_cache.shape != v_cache.shape:
        raise ValueError("q must be [B, Hq, d], the caches [B, Hkv, Lc, d] of one shape")
    if k_cache.shape[0] != q.shape[0] or k_cache.shape[3] != q.shape[2]:
        raise ValueError("the caches' B and d must match q's")
    if out is not None:
        _buf(out, "out", q.device, q.dtype, q.shape)
    if workspace is not None:
        _buf(workspace, "workspace", q.device, None)


def _check_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, out=None, lse=None, require_cuda=True):
    """q: [total_q, H, d]; k, v: [total_k, Hkv, d] of one shape; cu_seqlens:
    int32 [batch + 1] each."""
    torch = _torch()
    _inputs((q, k, v, cu_seqlens_q, cu_seqlens_k), q.device, require_cuda, "varlen tensors")
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or t.dim() != 3:
            raise ValueError("q, k, v must be [tokens, heads, d] bf16 tensors")
    if k.shape != v.shape or k.shape[2] != q.shape[2]:
        raise ValueError("k and v must be [total_k, Hkv, d] of one shape, d matching q's")
    for t in (cu_seqlens_q, cu_seqlens_k):
        if t.dtype != torch.int32 or t.dim() != 1:
            raise ValueError("cu_seqlens must be 1-D int32 tensors")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both hold batch + 1 >= 2 offsets")
    if out is not None:
        _buf(out, "out", q.device, q.dtype, q.shape)
    if lse is not None:
        _buf(lse, "lse", q.device, torch.float32, (q.shape[1], q.shape[0]))


def _raise(code, where):
    if code != 0:
        raise MalaError(code, where)


def default_tile(dtype) -> int:
    torch = _torch()
    return 128 if dtype == torch.bfloat16 else 64


def n_blocks(L: int, tile: int) -> int:
    return (L + tile - 1) // tile


def mala_fwd(q, k, v, tau: float = 1.0, tile: int | None = None, scale: float = 0.0,
             trace: bool = False, out=None, lse=None, o32=None, stream=None):
    """Forward pass. q, k, v: [B, H, L, d] (bf16 with d = 128, or float32).

    Returns (O, LSE) or, with ``trace=True``, (O, LSE, kept_tiles, keep_bits)
    where kept_tiles is int32 [B, H, nb] and keep_bits int32 [B, H, nb, nw].
    ``o32=True`` (or a float32 tensor shaped like q) also writes the float32
    output and appends it to the returned tuple (pass it to mala_bwd)."""
    torch = _check_prefill(q, k, v)
    B, H, L, d = q.shape
    tile = default_tile(q.dtype) if tile is None else tile
    o = torch.empty_like(q) if out is None else out
    lse_t = torch.empty((B, H, L), dtype=torch.float32, device=q.device) if lse is None else lse
    o32_t = None
    if o32 is True:
        o32_t = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    elif o32 is not None and o32 is not False:
        o32_t = o32
    _check_fwd_buffers(q, out=o, lse=lse_t, o32=o32_t)
    kept = bits = None
    if trace:
        nb = n_blocks(L, tile)
        kept = torch.empty((B, H, nb), dtype=torch.int32, device=q.device)
        bits = torch.empty((B, H, nb, (nb + 31) // 32), dtype=torch.int32, device=q.device)
    code = lib().mala_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse_t), _ptr(o32_t), B, H,
                          k.shape[1], L, d, _dtype_code(q), float(tau), int(tile), float(scale),
                          _ptr(kept), _ptr(bits), _stream(stream))
    _raise(code, "mala_fwd")
    res = (o, lse_t, kept, bits) if trace else (o, lse_t)
    return res + (o32_t,) if o32_t is not None else res


def mala_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                    tau: float = 1.0, scale: float = 0.0, trace: bool = False, out=None,
                    lse=None, stream=None):
    """Prefill of chunks appended to KV caches, sequences packed.
    q: [total_q, H, d] bf16; k, v: [total_k, Hkv, d] bf16; cu_seqlens_*:
    int32 CUDA tensors [batch + 1]. Returns (O [total_q, H, d], LSE [H,
    total_q]) or, with ``trace=True``, also kept_tiles [batch, H, nbq] and
    keep_bits [batch, H, nbq, nw] (bit k = key tile k)."""
    torch = _torch()
    _check_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, out=out, lse=lse)
    total_q, H, d = q.shape
    total_k, Hkv, _ = k.shape
    batch = cu_seqlens_q.numel() - 1
    o = torch.empty_like(q) if out is None else out
    lse_t = torch.empty((H, total_q), dtype=torch.float32, device=q.device) if lse is None else lse
    kept = bits = None
    if trace:
        nbq = n_blocks(max_seqlen_q, 128)
        nw = int(lib().mala_varlen_trace_words(max_seqlen_q, max_seqlen_k))
        kept = torch.zeros((batch, H, nbq), dtype=torch.int32, device=q.device)
        bits = torch.zeros((batch, H, nbq, nw), dtype=torch.int32, device=q.device)
    code = lib().mala_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse_t),
                                 _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), batch, int(max_seqlen_q),
                                 int(max_seqlen_k), total_q, total_k, H, Hkv, d, float(tau), 128,
                                 float(scale), _ptr(kept), _ptr(bits), _stream(stream))
    _raise(code, "mala_fwd_varlen")
    return (o, lse_t, kept, bits) if trace else (o, lse_t)


def bwd_workspace_bytes(B, H, L, d) -> int:
    return int(lib().mala_bwd_workspace_bytes(B, H, L, d))


def mala_bwd(q, k, v, o, do, lse, tau: float = 1.0, tile: int | None = None,
             scale: float = 0.0, trace: bool = False, workspace=None, grads=None, o32=None,
             stream=None):
    """Backward pass. Returns (dQ, dK, dV) or, with ``trace=True``,
    (dQ, dK, dV, kept_tiles [B, H, nb] per key block, keep_bits [B, H, nb, nw]).
    ``o32``: the float32 forward output (recommended for bf16), used for the
    row terms D = <dO, O>. Only O (or o32) and lse come from the forward."""
    torch = _check_prefill(q, k, v, o, do)
    B, H, L, d = q.shape
    tile = default_tile(q.dtype) if tile is None else tile
    if grads is None:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    else:
        dq, dk, dv = grads
    nbytes = bwd_workspace_bytes(B, H, L, d)
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device) if workspace is None \
        else workspace
    kept = bits = None
    if trace:
        nb = n_blocks(L, tile)
        kept = torch.empty((B, H, nb), dtype=torch.int32, device=q.device)
        bits = torch.empty((B, H, nb, (nb + 31) // 32), dtype=torch.int32, device=q.device)
    _check_bwd_buffers(q, k, lse, o32=o32, grads=(dq, dk, dv), workspace=ws)
    code = lib().mala_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(o32), _ptr(do), _ptr(lse),
                          _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
                          ws.numel() * ws.element_size(), B, H,
                          k.shape[1], L, d, _dtype_code(q),
                          float(tau), int(tile), float(scale), _ptr(kept), _ptr(bits),
                          _stream(stream))
    _raise(code, "mala_bwd")
    return (dq, dk, dv, kept, bits) if trace else (dq, dk, dv)


def decode_workspace_bytes(B, Hq, Hkv, Lc, d) -> int:
    return int(lib().mala_decode_workspace_bytes(B, Hq, Hkv, Lc, d))


def mala_decode(q, k_cache, v_cache, tau: float = 1.0, scale: float = 0.0, trace: bool = False,
                workspace=None, out=None, stream=None, per_head: bool = False):
    """One decode step. q: [B, Hq, d] bf16; caches: [B, Hkv, Lc, d] bf16.
    Returns o [B, Hq, d] or, with ``trace=True``, (o, kept_tiles [B, Hkv],
    keep_bits [B, Hkv, nw]); with ``per_head=True`` every query head applies
    the test alone and the trace is per query head ([B, Hq], [B, Hq, nw])."""
    torch = _torch()
    _check_decode(q, k_cache, v_cache, out=out, workspace=workspace)
    B, Hq, d = q.shape
    _, Hkv, Lc, _ = k_cache.shape
    o = torch.empty_like(q) if out is None else out
    nbytes = decode_workspace_bytes(B, Hq, Hkv, Lc, d)
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device) if workspace is None \
        else workspace
    kept = bits = None
    if trace:
        nt = n_blocks(Lc, 128)
        rows = Hq if per_head else Hkv
        kept = torch.empty((B, rows), dtype=torch.int32, device=q.device)
        bits = torch.empty((B, rows, (nt + 31) // 32), dtype=torch.int32, device=q.device)
    code = lib().mala_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), B, Hq, Hkv, Lc, d,
                             float(tau), float(scale), int(bool(per_head)), _ptr(ws),
                             ws.numel() * ws.element_size(),
                             _ptr(kept), _ptr(bits), _stream(stream))
    _raise(code, "mala_decode")
    return (o, kept, bits) if trace else o


NOALLOC_SCRATCH_BYTES = 8 << 20  # MALA_DECODE_NOALLOC_SCRATCH_BYTES in include/mala.h


def mala_decode_noalloc(q, k_cache, v_cache, tau: float = 1.0, scale: float = 0.0,
                        trace: bool = False, out=None, stream=None):
    """mala_decode without a workspace: the library's own static device array
    (NOALLOC_SCRATCH_BYTES, shared by every call on the device) serves as
    scratch, for callers that cannot allocate device memory. Calls that
    overlap on the GPU race on that array. Raises MalaError
    (MALA_ERR_TOO_LARGE) when the shape needs more scratch than the array
    holds. The output (and trace) tensors are the caller's: pass ``out`` to
    avoid allocating here too."""
    torch = _torch()
    _check_decode(q, k_cache, v_cache, out=out)
    B, Hq, d = q.shape
    _, Hkv, Lc, _ = k_cache.shape
    o = torch.empty_like(q) if out is None else out
    kept = bits = None
    if trace:
        nt = n_blocks(Lc, 128)
        kept = torch.empty((B, Hkv), dtype=torch.int32, device=q.device)
        bits = torch.empty((B, Hkv, (nt + 31) // 32), dtype=torch.int32, device=q.device)
    code = lib().mala_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), B, Hq, Hkv,
                                     Lc, d, float(tau), float(scale), _ptr(kept), _ptr(bits),
                                     _stream(stream))
    _raise(code, "mala_decode_noalloc")
    return (o, kept, bits) if trace else o


def mala_check(stream=None):
    """Synchronize the stream and raise MalaError if a kernel reported a
    timeout or the stream holds a CUDA error."""
    _raise(lib().mala_check(_stream(stream)), "mala_check")


def mala_selftest_wait(stream=None):
    """Diagnostic of the timeout path: one device thread waits, with the
    kernels' bounded wait (about two seconds), on a barrier nothing arrives
    on, so the next mala_check raises MalaError (MALA_ERR_TIMEOUT) once."""
    _raise(lib().mala_selftest_wait(_stream(stream)), "mala_selftest_wait")


def unpack_bits(bits, n: int):
    """[..., nw] int32 keep bitmask -> [..., n] uint8 (host numpy)."""
    import numpy as np
    b = bits.cpu().numpy().astype(np.uint32)
    shifts = np.arange(32, dtype=np.uint32)
    out = ((b[..., :, None] >> shifts) & 1).astype(np.uint8)
    return out.reshape(*b.shape[:-1], -1)[..., :n]
