"""The C ABI without a GPU: the library loads, exports every call that
include/mala.h declares, and rejects bad arguments on the host before any
CUDA call."""

import ctypes
import os
import re

import pytest

import mass_adaptive_causal_b200 as mala

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mala.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mala_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from mass_adaptive_causal_b200 import build
    build.build()
    return mala.lib()


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert {"mala_fwd", "mala_bwd", "mala_decode", "mala_check"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code, name in mala.STATUS.items():
        assert lib.mala_status_string(code).decode() == name
    assert lib.mala_version() >= 100


def _fwd(lib, ptrs=(16, 16, 16, 16, 16, 0), B=1, H=1, L=256, d=128, dt=1, tau=1.0, tile=128,
         Hkv=None):
    p = [ctypes.c_void_p(x) if x else None for x in ptrs]
    return lib.mala_fwd(*p, B, H, H if Hkv is None else Hkv, L, d, dt, tau, tile, 0.0, None, None,
                        None)


def test_fwd_argument_checks(lib):
    assert _fwd(lib, tau=-1.0) == 1
    assert _fwd(lib, tau=float("nan")) == 1
    assert _fwd(lib, tau=float("inf")) == 1
    assert _fwd(lib, B=0) == 1
    assert _fwd(lib, L=-1) == 1
    assert _fwd(lib, d=64) == 2                 # bf16 needs d = 128
    assert _fwd(lib, tile=64) == 2              # bf16 needs tile 128
    assert _fwd(lib, dt=0, d=64, tile=128) == 2  # f32 tile is 64
    assert _fwd(lib, dt=0, d=48, tile=64) == 2
    assert _fwd(lib, dt=7) == 2
    assert _fwd(lib, ptrs=(0, 16, 16, 16, 16, 0)) == 1
    assert _fwd(lib, ptrs=(16, 16, 8, 16, 16, 0)) == 1  # misaligned
    assert _fwd(lib, ptrs=(16, 16, 16, 16, 16, 8)) == 1  # misaligned float32 output
    assert _fwd(lib, L=0) == 0                   # empty input: nothing to do
    assert _fwd(lib, B=300, H=300) == 1          # grid limit
    assert _fwd(lib, H=4, Hkv=3) == 1            # query heads not a multiple of kv heads
    assert _fwd(lib, H=4, Hkv=0) == 1
    assert _fwd(lib, H=4, Hkv=2, dt=0, d=64, tile=64) == 2  # grouped heads: bf16 only
    assert _fwd(lib, H=4, Hkv=2, L=0) == 0


def test_bwd_and_decode_argument_checks(lib):
    v = ctypes.c_void_p(256)
    need = lib.mala_bwd_workspace_bytes(1, 2, 1000, 128)
    r256 = lambda x: ((x + 255) // 256) * 256
    nb64 = (1000 + 63) // 64
    assert need == (r256(2 * 1000 * 4) + r256(2 * 1000 * 128 * 4)
                    + r256(2 * nb64 * ((nb64 + 31) // 32) * 4) + 256)  # + the column counter
    args = [v] * 11
    assert lib.mala_bwd(*args, need - 1, 1, 2, 2, 1000, 128, 1, 1.0, 128, 0.0, None, None, None) == 1
    assert lib.mala_bwd(*args, need, 1, 2, 2, 1000, 128, 1, -0.5, 128, 0.0, None, None, None) == 1
    assert lib.mala_bwd(*args, need, 1, 2, 2, 0, 128, 1, 1.0, 128, 0.0, None, None, None) == 0
    assert lib.mala_bwd(*args, need, 1, 2, 3, 1000, 128, 1, 1.0, 128, 0.0, None, None, None) == 1
    ws = lib.mala_decode_workspace_bytes(2, 8, 2, 1000, 128)
    assert ws > 0
    dec = lambda Hq, Hkv, d, tau, nbytes, ph=0: lib.mala_decode(v, v, v, v, 2, Hq, Hkv, 1000, d,
                                                                tau, 0.0, ph, v, nbytes, None,
                                                                None, None)
    assert dec(8, 3, 128, 1.0, ws) == 1    # Hq % Hkv
    assert dec(8, 2, 64, 1.0, ws) == 2     # d
    assert dec(32, 2, 128, 1.0, 1 << 30) == 2  # group of 16 heads > 8
    assert dec(8, 2, 128, -1.0, ws) == 1
    assert dec(8, 2, 128, 1.0, ws - 1) == 1
    assert dec(8, 2, 128, 1.0, ws, ph=2) == 1   # per_head is 0 or 1


def test_python_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(mala, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(mala, "_lib", None)
    with pytest.raises(RuntimeError):
        mala.lib()


def test_decode_noalloc_argument_checks(lib):
    """Shape checks, including the scratch limit, come before any CUDA call."""
    p = [ctypes.c_void_p(16)] * 4
    f = lib.mala_decode_noalloc
    assert f(*p, 1, 8, 2, 1000, 128, -1.0, 0.0, None, None, None) == 1
    assert f(*p, 1, 8, 3, 1000, 128, 1.0, 0.0, None, None, None) == 1
    assert f(*p, 1, 8, 2, 1000, 64, 1.0, 0.0, None, None, None) == 2
    assert f(*p, 1, 32, 2, 1000, 128, 1.0, 0.0, None, None, None) == 2
    assert f(None, *p[1:], 1, 8, 2, 1000, 128, 1.0, 0.0, None, None, None) == 1
    B, Hq, Hkv, Lc, d = 64, 64, 8, 32768, 128
    assert mala.decode_workspace_bytes(B, Hq, Hkv, Lc, d) > mala.NOALLOC_SCRATCH_BYTES
    assert f(*p, B, Hq, Hkv, Lc, d, 1.0, 0.0, None, None, None) == 5
    assert lib.mala_status_string(5).decode() == "MALA_ERR_TOO_LARGE"


def test_fwd_varlen_argument_checks(lib):
    v = ctypes.c_void_p(256)
    f = lambda batch=2, mq=100, mk=200, tq=150, tk=300, H=2, Hkv=1, d=128, tau=1.0, tile=128: \
        lib.mala_fwd_varlen(v, v, v, v, v, v, v, batch, mq, mk, tq, tk, H, Hkv, d, tau, tile, 0.0,
                            None, None, None)
    assert f(batch=0) == 1
    assert f(H=3, Hkv=2) == 1
    assert f(tau=-1.0) == 1
    assert f(d=64) == 2
    assert f(tile=64) == 2
    assert f(tq=0) == 0
    assert lib.mala_fwd_varlen(None, v, v, v, v, v, v, 2, 100, 200, 150, 300, 2, 1, 128, 1.0, 128,
                               0.0, None, None, None) == 1
    assert lib.mala_varlen_trace_words(100, 200) == 1
    assert lib.mala_varlen_trace_words(4096, 131072) == (32 + 1024 + 31) // 32


def test_header_is_c_and_the_library_links_from_c(lib, tmp_path):
    """A C11 program (tests/c/abi_host.c) includes include/mala.h, links
    libmala.so and checks the calls that need no GPU."""
    import subprocess
    src = os.path.join(ROOT, "tests", "c", "abi_host.c")
    exe = tmp_path / "abi_host"
    libdir = os.path.dirname(mala.LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I",
                    os.path.join(ROOT, "include"), src, "-o", str(exe), f"-L{libdir}",
                    f"-Wl,-rpath,{libdir}", "-l:libmala.so"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"
