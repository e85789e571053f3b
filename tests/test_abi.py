"""The C-ABI library builds, loads and exports every symbol include/kda.h declares.

These run without a GPU: they only call entry points on argument errors that
the library rejects on the host before touching CUDA.
"""
import ctypes
import os
import re
import subprocess

import pytest

import gated_delta_rule_109_b200 as kda
from gated_delta_rule_109_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]


def declared_functions():
    names = []
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"\b(kda_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"kda_forward", "kda_decode_step", "kda_status_string", "kda_check_status"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", kbuild.LIB], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(\w+)$", out, flags=re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(lib, n)
    assert set(kda.EXPORTS) == set(names)


def test_library_is_built_for_sm100a():
    out = subprocess.run(["strings", kbuild.LIB], capture_output=True, text=True).stdout
    assert "sm_100a" in out


def test_status_strings(lib):
    for code, name in enumerate(["KDA_OK", "KDA_ERR_INVALID_ARG", "KDA_ERR_UNSUPPORTED",
                                 "KDA_ERR_MISALIGNED", "KDA_ERR_CUDA", "KDA_ERR_TIMEOUT"]):
        assert lib.kda_status_string(code).decode() == name
    assert lib.kda_status_string(99).decode() == "KDA_ERR_UNKNOWN"
    assert lib.kda_version() >= 100


FAKE = 0x100000          # 16-byte aligned, never dereferenced: every call below fails validation


def _fwd(lib, q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, s0=None, out=FAKE, sT=None,
         B=1, T=8, H=2, dk=128, dv=128, dtype=kda.KDA_BF16, scale=0.0):
    return lib.kda_forward(q, k, v, la, beta, s0, out, sT, B, T, H, dk, dv, dtype,
                           ctypes.c_float(scale), None)


def _dec(lib, q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, st=FAKE, out=FAKE,
         B=1, H=2, dk=128, dv=128, dtype=kda.KDA_BF16, scale=0.0):
    return lib.kda_decode_step(q, k, v, la, beta, st, out, B, H, dk, dv, dtype,
                               ctypes.c_float(scale), None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), kda.KDA_ERR_INVALID_ARG),
    (dict(k=None), kda.KDA_ERR_INVALID_ARG),
    (dict(v=None), kda.KDA_ERR_INVALID_ARG),
    (dict(la=None), kda.KDA_ERR_INVALID_ARG),
    (dict(beta=None), kda.KDA_ERR_INVALID_ARG),
    (dict(out=None), kda.KDA_ERR_INVALID_ARG),
    (dict(B=0), kda.KDA_ERR_INVALID_ARG),
    (dict(H=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(T=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=0), kda.KDA_ERR_INVALID_ARG),
    (dict(dtype=7), kda.KDA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), kda.KDA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=96), kda.KDA_ERR_UNSUPPORTED),
    (dict(dv=256), kda.KDA_ERR_UNSUPPORTED),
    (dict(q=FAKE + 8), kda.KDA_ERR_MISALIGNED),
    (dict(v=FAKE + 2), kda.KDA_ERR_MISALIGNED),
    (dict(la=FAKE + 4), kda.KDA_ERR_MISALIGNED),
    (dict(out=FAKE + 4), kda.KDA_ERR_MISALIGNED),
    (dict(beta=FAKE + 2), kda.KDA_ERR_MISALIGNED),
    (dict(s0=FAKE + 4), kda.KDA_ERR_MISALIGNED),
    (dict(sT=FAKE + 8), kda.KDA_ERR_MISALIGNED),
])
def test_forward_rejects_bad_arguments_before_launch(lib, kw, code):
    assert _fwd(lib, **kw) == code


def test_forward_empty_sequence_without_state_is_a_no_op(lib):
    # T = 0 and no final state: nothing to do, nothing touched, no CUDA call
    assert _fwd(lib, q=None, k=None, v=None, la=None, beta=None, out=None, T=0) == kda.KDA_OK
    # T = 0 with final_state aliasing initial_state: also nothing to do
    assert _fwd(lib, q=None, k=None, v=None, la=None, beta=None, out=None, T=0,
                s0=FAKE, sT=FAKE) == kda.KDA_OK


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), kda.KDA_ERR_INVALID_ARG),
    (dict(st=None), kda.KDA_ERR_INVALID_ARG),
    (dict(out=None), kda.KDA_ERR_INVALID_ARG),
    (dict(B=0), kda.KDA_ERR_INVALID_ARG),
    (dict(dtype=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=32), kda.KDA_ERR_UNSUPPORTED),
    (dict(st=FAKE + 4), kda.KDA_ERR_MISALIGNED),
    (dict(k=FAKE + 2), kda.KDA_ERR_MISALIGNED),
])
def test_decode_rejects_bad_arguments_before_launch(lib, kw, code):
    assert _dec(lib, **kw) == code


def test_binding_raises_when_library_missing(tmp_path):
    with pytest.raises(RuntimeError, match="not built"):
        kda.load(str(tmp_path / "libkda.so"))


def test_binding_error_carries_status(lib):
    err = kda.KDAError(kda.KDA_ERR_UNSUPPORTED, "kda_forward")
    assert err.status == kda.KDA_ERR_UNSUPPORTED and "KDA_ERR_UNSUPPORTED" in str(err)
