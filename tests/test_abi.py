"""The C-ABI library: it loads, it exports every entry point the header
declares, and argument errors come back as status codes before anything
touches a GPU (these calls never reach the CUDA runtime)."""
import ctypes
import os
import re

import pytest

from sparse_long_sequence_fwd_b200 import build, lf_attn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lf_attn.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return lf_attn.load()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lf_attn_\w+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_symbols() == sorted(lf_attn.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_strerror_and_workspace(lib):
    for code in range(6):
        assert lf_attn.strerror(code)
    assert lib.lf_attn_workspace_bytes(1, 12, 4096, 64, 1, 1) > 0
    assert lib.lf_attn_workspace_bytes(0, 12, 4096, 64, 1, 1) == 0
    # f16 uses the tensor-core path's workspace, the same as bf16
    assert lib.lf_attn_workspace_bytes(2, 12, 4096, 64, 64, 2) == lib.lf_attn_workspace_bytes(2, 12, 4096, 64, 64, 1)


FAKE = 1 << 20  # aligned non-null address, never dereferenced by the argument checks
P = ctypes.c_void_p


def _call(lib, **kw):
    a = dict(q=P(FAKE), k=P(FAKE), v=P(FAKE), out=P(FAKE), B=1, H=2, T=64, d=64, r=4, dil=None, g=None,
             ng=0, pad=None, scale=0.125, dtype=1, stream=None)
    a.update(kw)
    return lib.lf_attn_fwd(a["q"], a["k"], a["v"], a["out"], a["B"], a["H"], a["T"], a["d"], a["r"], a["dil"],
                           a["g"], a["ng"], a["pad"], a["scale"], a["dtype"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(out=None), 1), (dict(B=0), 1), (dict(H=-1), 1), (dict(T=0), 1),
    (dict(d=0), 1), (dict(r=-1), 1), (dict(ng=-1), 1), (dict(ng=2), 1),          # n_global > 0 needs global_idx
    (dict(g=P(FAKE), ng=0), 1), (dict(scale=float("nan")), 1), (dict(dtype=7), 1),
    (dict(q=P(FAKE + 2)), 1),                                                    # misaligned
    (dict(dil=(ctypes.c_int32 * 2)(1, 0)), 1),                                   # dilation < 1
    (dict(B=1 << 20, H=1 << 20, T=1 << 20), 1),                                  # size overflow
    (dict(d=32), 2), (dict(d=96), 2), (dict(d=256), 2),                          # bf16 path: d == 64 or 128
    (dict(dil=(ctypes.c_int32 * 2)(1, 9)), 2),                                   # TMA element stride <= 8
    (dict(T=(1 << 20) + 1), 2), (dict(H=129), 2), (dict(dtype=0, d=129), 2),
    (dict(dtype=2, d=32), 2), (dict(dtype=2, dil=(ctypes.c_int32 * 2)(1, 9)), 2),  # f16: same limits as bf16
    (dict(dtype=3), 1),
])
def test_argument_errors_return_status_without_launch(lib, kw, code):
    assert _call(lib, **kw) == code


def test_too_many_dilation_kinds(lib):
    dil = (ctypes.c_int32 * 5)(1, 2, 3, 4, 5)
    assert _call(lib, H=5, dil=dil) == 2


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(lf_attn, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(lf_attn, "_lib", None)
    with pytest.raises(RuntimeError):
        lf_attn.load()



def _call_rand(lib, n_rand=2, rb=P(FAKE), **kw):
    a = dict(q=P(FAKE), k=P(FAKE), v=P(FAKE), out=P(FAKE), B=1, H=2, T=64, d=64, r=4, dil=None, g=None,
             ng=0, pad=None, scale=0.125, dtype=1, stream=None)
    a.update(kw)
    return lib.lf_attn_fwd_rand(a["q"], a["k"], a["v"], a["out"], a["B"], a["H"], a["T"], a["d"], a["r"], a["dil"],
                                a["g"], a["ng"], a["pad"], a["scale"], a["dtype"], rb, n_rand, a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(n_rand=5), 1), (dict(n_rand=-1), 1), (dict(rb=None), 1), (dict(n_rand=0), 1),  # table iff draws
    (dict(rb=P(FAKE + 2)), 1),                                                          # misaligned table
    (dict(dtype=0), 2), (dict(d=128), 2), (dict(dil=(ctypes.c_int32 * 2)(1, 2)), 2),   # bf16/f16, d 64, dil 1
])
def test_random_block_argument_errors(lib, kw, code):
    assert _call_rand(lib, **kw) == code
