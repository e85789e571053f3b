"""The C-ABI library builds, loads and exports every symbol include/kda.h declares.

These run without a GPU: they only call entry points on argument errors that
the library rejects on the host before touching CUDA.
"""
import ctypes
import os
import re
import subprocess

import pytest
import torch

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


def test_every_compile_and_the_link_target_sm100a_only(monkeypatch, tmp_path):
    # the build's own command lines, recorded instead of run: one target, sm_100a
    cmds = []

    class Done:
        returncode, stdout, stderr = 0, "", ""

    monkeypatch.setattr(kbuild.subprocess, "run", lambda cmd, **kw: (cmds.append(cmd), Done())[1])
    monkeypatch.setattr(kbuild.os, "replace", lambda a, b: None)
    monkeypatch.setattr(kbuild, "BUILD", str(tmp_path))
    kbuild.build(force=True)
    assert len(cmds) == len(kbuild._sources()) + 1            # every kernel source, then the link
    for c in cmds:
        assert c.count("-gencode") == 1
        assert c[c.index("-gencode") + 1] == "arch=compute_100a,code=sm_100a"
    assert all("-c" in c for c in cmds[:-1]) and "-shared" in cmds[-1]


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
    # B * H beyond what the decode grid (several CTAs per head) can address
    (dict(B=1 << 15, H=1 << 15), kda.KDA_ERR_INVALID_ARG),
    (dict(B=(1 << 29) + 1, H=1), kda.KDA_ERR_INVALID_ARG),
])
def test_decode_rejects_bad_arguments_before_launch(lib, kw, code):
    assert _dec(lib, **kw) == code


def test_binding_raises_when_library_missing(tmp_path):
    with pytest.raises(RuntimeError, match="not built"):
        kda.load(str(tmp_path / "libkda.so"))


def test_binding_error_carries_status(lib):
    err = kda.KDAError(kda.KDA_ERR_UNSUPPORTED, "kda_forward")
    assert err.status == kda.KDA_ERR_UNSUPPORTED and "KDA_ERR_UNSUPPORTED" in str(err)


def _gdn(lib, q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, s0=None, out=FAKE, sT=None,
         B=1, T=8, H=2, dk=128, dv=128, dtype=kda.KDA_BF16, scale=0.0):
    return lib.kda_gdn_forward(q, k, v, la, beta, s0, out, sT, B, T, H, dk, dv, dtype,
                               ctypes.c_float(scale), None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), kda.KDA_ERR_INVALID_ARG),
    (dict(beta=None), kda.KDA_ERR_INVALID_ARG),
    (dict(B=0), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=96), kda.KDA_ERR_UNSUPPORTED),
    (dict(la=FAKE + 2), kda.KDA_ERR_MISALIGNED),      # the scalar gate needs 4-byte alignment only
    (dict(v=FAKE + 8), kda.KDA_ERR_MISALIGNED),
])
def test_gdn_forward_rejects_bad_arguments_before_launch(lib, kw, code):
    assert _gdn(lib, **kw) == code


def test_gdn_decode_rejects_bad_arguments_before_launch(lib):
    call = lambda **kw: lib.kda_gdn_decode_step(kw.get("q", FAKE), FAKE, FAKE, kw.get("la", FAKE), FAKE,
                                                kw.get("st", FAKE), FAKE, 1, 2, 128, 128, kda.KDA_BF16,
                                                ctypes.c_float(0.0), None)
    assert call(q=None) == kda.KDA_ERR_INVALID_ARG
    assert call(st=FAKE + 4) == kda.KDA_ERR_MISALIGNED
    assert call(la=FAKE + 1) == kda.KDA_ERR_MISALIGNED


def test_workspace_sizes(lib):
    full = lambda *a: lib.kda_forward_workspace_bytes(*a)
    mini = lambda *a: lib.kda_forward_workspace_min_bytes(*a)
    rec = full(1, 64, 1, 128, 128, kda.KDA_BF16)      # bytes of one chunk record (b, h, chunk)
    assert rec % 256 == 0 or rec % 16 == 0
    assert 140_000 < rec < 160_000
    assert full(4, 16384, 32, 128, 128, kda.KDA_BF16) == 128 * 256 * rec      # many heads: whole sequence
    assert full(2, 65, 3, 128, 128, kda.KDA_BF16) == 6 * 2 * rec             # ragged tail: 2 chunks
    assert mini(2, 65, 3, 128, 128, kda.KDA_BF16) == 6 * rec + 6 * 128 * 128 * 4
    assert mini(2, 64, 3, 128, 128, kda.KDA_BF16) == full(2, 64, 3, 128, 128, kda.KDA_BF16) == 6 * rec
    for args in [(1, 100, 2, 64, 64, kda.KDA_BF16), (1, 100, 2, 128, 128, kda.KDA_F32),
                 (1, 0, 2, 128, 128, kda.KDA_BF16), (0, 10, 2, 128, 128, kda.KDA_BF16)]:
        assert full(*args) == 0 and mini(*args) == 0
    # few heads and a long sequence: the pipelined schedule's two slots of 64 chunks
    # and the carried state, far less than the whole sequence's records
    state32 = 32 * 128 * 128 * 4
    assert kda.workspace_bytes(1, 65536, 32, 128, 128) == 2 * 64 * 32 * rec + state32
    assert kda.workspace_bytes(1, 8192, 32, 128, 128) == 2 * 64 * 32 * rec + state32
    assert kda.workspace_bytes(1, 8128, 32, 128, 128) == 32 * 127 * rec            # under 128 chunks
    # segments keep every record of the segment
    seg = lambda *a: lib.kda_segment_workspace_bytes(*a)
    assert seg(1, 65536, 32, 128, 128, kda.KDA_BF16) == 32 * 1024 * rec
    assert kda.workspace_bytes(1, 8192, 32, 128, 128, segment=True) == 32 * 128 * rec
    assert seg(1, 100, 2, 64, 64, kda.KDA_BF16) == 0


def test_forward_ws_validates_like_forward(lib):
    def fws(ws=FAKE * 16, nbytes=1 << 30, **kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, s0=None, out=FAKE, sT=None)
        a.update(kw)
        return lib.kda_forward_ws(a["q"], a["k"], a["v"], a["la"], a["beta"], a["s0"], a["out"], a["sT"],
                                  1, 8, 2, 128, 128, kda.KDA_BF16, ctypes.c_float(0.0), ws, nbytes, None)
    assert fws(q=None) == kda.KDA_ERR_INVALID_ARG
    assert fws(ws=FAKE + 16) == kda.KDA_ERR_MISALIGNED    # workspace must be 256-byte aligned
    assert fws(la=FAKE + 4) == kda.KDA_ERR_MISALIGNED


def test_segment_calls_validate_before_launch(lib):
    WS = FAKE * 16

    def local(T=8, transfer=FAKE, sT=FAKE, ws=WS, nbytes=1 << 40, dtype=kda.KDA_BF16, **kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, s0=None, out=FAKE)
        a.update(kw)
        return lib.kda_segment_local(a["q"], a["k"], a["v"], a["la"], a["beta"], a["s0"], a["out"], sT, transfer,
                                     1, T, 2, 128, 128, dtype, ctypes.c_float(0.0), ws, nbytes, None)
    assert local(T=0) == kda.KDA_ERR_INVALID_ARG
    assert local(transfer=None) == kda.KDA_ERR_INVALID_ARG
    assert local(sT=None) == kda.KDA_ERR_INVALID_ARG
    assert local(q=None) == kda.KDA_ERR_INVALID_ARG
    assert local(transfer=FAKE + 4) == kda.KDA_ERR_MISALIGNED
    assert local(la=FAKE + 4) == kda.KDA_ERR_MISALIGNED
    assert local(ws=WS + 16) == kda.KDA_ERR_MISALIGNED
    assert local(dtype=kda.KDA_F32) == kda.KDA_ERR_UNSUPPORTED
    assert local(ws=None) == kda.KDA_ERR_UNSUPPORTED
    assert local(nbytes=kda.workspace_bytes(1, 8, 2, 128, 128) - 1) == kda.KDA_ERR_UNSUPPORTED

    def start(R=2, P=FAKE, F=FAKE, S=FAKE, dk=128):
        return lib.kda_segment_start_state(P, F, R, S, 1, 2, dk, 128, None)
    assert start(R=0) == kda.KDA_ERR_INVALID_ARG
    assert start(P=None) == kda.KDA_ERR_INVALID_ARG
    assert start(dk=64) == kda.KDA_ERR_UNSUPPORTED
    assert start(S=FAKE + 4) == kda.KDA_ERR_MISALIGNED

    def correct(T=8, ws=WS, nbytes=1 << 40, sT=FAKE, out=FAKE):
        return lib.kda_segment_correct(FAKE, FAKE, out, sT, 1, T, 2, 128, 128, ws, nbytes, None)
    assert correct(T=0) == kda.KDA_ERR_INVALID_ARG
    assert correct(ws=None) == kda.KDA_ERR_INVALID_ARG
    assert correct(ws=WS + 16) == kda.KDA_ERR_MISALIGNED
    assert correct(out=FAKE + 4) == kda.KDA_ERR_MISALIGNED
    assert correct(sT=FAKE + 8) == kda.KDA_ERR_MISALIGNED
    assert correct(nbytes=kda.workspace_bytes(1, 8, 2, 128, 128) - 1) == kda.KDA_ERR_UNSUPPORTED


def test_backward_validates_before_launch(lib):
    WS = FAKE * 16

    def bwd(T=8, dk=128, dv=128, dtype=kda.KDA_BF16, ws=WS, nbytes=1 << 40, scale=0.0, **kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, s0=None, go=FAKE, gs=None, gq=FAKE, gk=FAKE,
                 gv=FAKE, gla=FAKE, gb=FAKE, gs0=FAKE)
        a.update(kw)
        return lib.kda_backward(a["q"], a["k"], a["v"], a["la"], a["beta"], a["s0"], a["go"], a["gs"], a["gq"],
                                a["gk"], a["gv"], a["gla"], a["gb"], a["gs0"], 1, T, 2, dk, dv, dtype,
                                ctypes.c_float(scale), ws, nbytes, None)
    assert bwd(q=None) == kda.KDA_ERR_INVALID_ARG
    assert bwd(go=None) == kda.KDA_ERR_INVALID_ARG
    assert bwd(gla=None) == kda.KDA_ERR_INVALID_ARG
    assert bwd(ws=None) == kda.KDA_ERR_INVALID_ARG
    assert bwd(T=-1) == kda.KDA_ERR_INVALID_ARG
    assert bwd(dtype=5) == kda.KDA_ERR_INVALID_ARG
    assert bwd(scale=float("nan")) == kda.KDA_ERR_INVALID_ARG
    assert bwd(nbytes=kda.backward_workspace_bytes(1, 8, 2, 128, 128) - 1) == kda.KDA_ERR_INVALID_ARG
    assert bwd(dk=96, dv=96) == kda.KDA_ERR_UNSUPPORTED
    assert bwd(dk=64, dv=128) == kda.KDA_ERR_UNSUPPORTED
    assert bwd(q=FAKE + 8) == kda.KDA_ERR_MISALIGNED
    assert bwd(gk=FAKE + 4) == kda.KDA_ERR_MISALIGNED
    assert bwd(beta=FAKE + 2) == kda.KDA_ERR_MISALIGNED
    assert bwd(ws=WS + 16) == kda.KDA_ERR_MISALIGNED
    assert bwd(s0=FAKE + 4) == kda.KDA_ERR_MISALIGNED
    # T = 0 without a wanted initial-state gradient: nothing to do, no CUDA call
    assert bwd(T=0, q=None, k=None, v=None, la=None, beta=None, go=None, gq=None, gk=None, gv=None, gla=None,
               gb=None, gs0=None, ws=None) == kda.KDA_OK
    wb = lib.kda_backward_workspace_bytes
    assert wb(1, 65, 2, 128, 128) == (9 + 2) * 2 * 128 * 128 * 4
    assert wb(3, 64, 5, 64, 64) == (8 + 1) * 15 * 64 * 64 * 4
    assert wb(1, 0, 2, 128, 128) == 0 and wb(1, 64, 2, 96, 96) == 0 and wb(1, 64, 2, 64, 128) == 0


def test_gdn_forward_ws_validates_like_gdn_forward(lib):
    def g(ws=FAKE * 16, nbytes=1 << 30, la=FAKE, **kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, beta=FAKE, s0=None, out=FAKE, sT=None)
        a.update(kw)
        return lib.kda_gdn_forward_ws(a["q"], a["k"], a["v"], la, a["beta"], a["s0"], a["out"], a["sT"],
                                      1, 8, 2, 128, 128, kda.KDA_BF16, ctypes.c_float(0.0), ws, nbytes, None)
    assert g(q=None) == kda.KDA_ERR_INVALID_ARG
    assert g(ws=FAKE + 16) == kda.KDA_ERR_MISALIGNED      # workspace must be 256-byte aligned
    assert g(la=FAKE + 2) == kda.KDA_ERR_MISALIGNED       # the scalar gate needs 4-byte alignment
    assert g(v=FAKE + 8) == kda.KDA_ERR_MISALIGNED


def test_forward_host_validates_before_any_copy(lib):
    WS = FAKE * 16

    def fh(T=8, ws=WS, nbytes=1 << 40, block=0, dk=128, dtype=kda.KDA_BF16, **kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, s0=None, out=FAKE, sT=None)
        a.update(kw)
        return lib.kda_forward_host(a["q"], a["k"], a["v"], a["la"], a["beta"], a["s0"], a["out"], a["sT"],
                                    1, T, 2, dk, 128, dtype, ctypes.c_float(0.0), block, ws, nbytes, None)
    assert fh(q=None) == kda.KDA_ERR_INVALID_ARG
    assert fh(out=None) == kda.KDA_ERR_INVALID_ARG
    assert fh(ws=None) == kda.KDA_ERR_INVALID_ARG
    assert fh(block=-1) == kda.KDA_ERR_INVALID_ARG
    assert fh(T=-1) == kda.KDA_ERR_INVALID_ARG
    assert fh(dtype=9) == kda.KDA_ERR_INVALID_ARG
    assert fh(dk=96) == kda.KDA_ERR_UNSUPPORTED
    assert fh(ws=WS + 16) == kda.KDA_ERR_MISALIGNED
    need = lib.kda_forward_host_workspace_bytes(1, 8, 2, 128, 128, kda.KDA_BF16, 0)
    assert need > 0 and fh(nbytes=need - 1) == kda.KDA_ERR_INVALID_ARG
    # the workspace grows with the block length, not with T beyond one block
    wb = lambda T, blk: lib.kda_forward_host_workspace_bytes(1, T, 32, 128, 128, kda.KDA_BF16, blk)
    assert wb(65536, 4096) == wb(8192, 4096) < wb(65536, 8192)
    assert wb(64, 0) == wb(64, 8192) and lib.kda_forward_host_workspace_bytes(1, 8, 2, 96, 96, kda.KDA_BF16, 0) == 0


def test_header_is_plain_c_and_links(lib, tmp_path):
    """include/kda.h compiles as pedantic C99, and a C program links libkda.so and
    calls host-only entry points (no GPU needed)."""
    src = tmp_path / "use_kda.c"
    src.write_text('#include <stdio.h>\n#include <string.h>\n#include "kda.h"\n'
                   'int main(void) {\n'
                   '  if (kda_version() < 300) return 1;\n'
                   '  if (strcmp(kda_status_string(KDA_ERR_TIMEOUT), "KDA_ERR_TIMEOUT") != 0) return 2;\n'
                   '  if (kda_forward_workspace_bytes(1, 64, 1, 128, 128, KDA_BF16) == 0) return 3;\n'
                   '  if (kda_forward(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, 8, 1, 128, 128,\n'
                   '                  KDA_BF16, 0.0f, NULL) != KDA_ERR_INVALID_ARG) return 4;\n'
                   '  puts("ok");\n  return 0;\n}\n')
    exe = tmp_path / "use_kda"
    libdir = os.path.dirname(kbuild.LIB)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-lkda", "-Wl,-rpath," + libdir], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)


def _host_prefill(B=1, T=8, H=2, d=128):
    q = torch.zeros((B, T, H, d), dtype=torch.bfloat16)
    return dict(q=q, k=q.clone(), v=q.clone(), log_alpha=torch.zeros((B, T, H, d)), beta=torch.zeros((B, T, H)))


def test_binding_refuses_host_tensors_before_any_device_work(lib):
    # the kernels take device memory only: host tensors are refused in the binding
    x = _host_prefill()
    args = (x["q"], x["k"], x["v"], x["log_alpha"], x["beta"])
    for call in (lambda: kda.forward(*args), lambda: kda.gdn_forward(x["q"], x["k"], x["v"], None, x["beta"]),
                 lambda: kda.forward_noalloc(*args),
                 lambda: kda.backward(*args, torch.zeros((1, 8, 2, 128))),
                 lambda: kda.segment_local(*args, workspace=torch.empty(16, dtype=torch.uint8)),
                 lambda: kda.segment_start_state(torch.zeros((1, 1, 2, 128, 128)), torch.zeros((1, 1, 2, 128, 128))),
                 lambda: kda.segment_correct(torch.zeros((1, 2, 128, 128)), torch.zeros((1, 2, 128, 128)),
                                             torch.zeros((1, 8, 2, 128)), workspace=torch.empty(16, dtype=torch.uint8)),
                 lambda: kda.forward_raw(*args, workspace=torch.empty(16, dtype=torch.uint8))):
        with pytest.raises(ValueError, match="CUDA tensors"):
            call()
    q1 = torch.zeros((1, 2, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensors"):
        kda.decode_step(q1, q1, q1, torch.zeros((1, 2, 128)), torch.zeros((1, 2)), torch.zeros((1, 2, 128, 128)))


def test_binding_refuses_a_workspace_off_the_device(lib):
    dev = torch.device("cuda", 0)
    with pytest.raises(TypeError):
        kda._need_workspace(object(), dev, "kda_forward_ws")
    with pytest.raises(ValueError, match="contiguous CUDA tensor"):
        kda._need_workspace(torch.empty(64, dtype=torch.uint8), dev, "kda_forward_ws")
    with pytest.raises(ValueError, match="contiguous CUDA tensor"):
        kda._need_workspace(torch.empty((8, 8), dtype=torch.uint8).t(), dev, "kda_forward_ws")
    # the host-buffer prefill: host inputs, but its workspace must be device memory
    x = _host_prefill()
    with pytest.raises(ValueError, match="contiguous CUDA tensor"):
        kda.forward_host(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], out=torch.empty((1, 8, 2, 128)),
                         final_state=torch.empty((1, 2, 128, 128)), workspace=torch.empty(64, dtype=torch.uint8),
                         device="cuda:0")


def test_forward_host_empty_sequence_copies_the_state_on_the_host(lib):
    # T = 0 touches no device: the final state is the initial state (or zeros), in host memory
    import numpy as np
    s0 = np.arange(2 * 64 * 64, dtype=np.float32).reshape(1, 2, 64, 64)
    fin = np.full_like(s0, 7.0)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    call = lambda s_in, s_out: lib.kda_forward_host(None, None, None, None, None, s_in, None, s_out, 1, 0, 2, 64, 64,
                                                   kda.KDA_F32, ctypes.c_float(0.0), 0, None, 0, None)
    assert call(p(s0), p(fin)) == kda.KDA_OK and np.array_equal(fin, s0)
    assert call(None, p(fin)) == kda.KDA_OK and not fin.any()
    assert call(p(s0), p(s0)) == kda.KDA_OK and s0[0, 1, 63, 63] == 2 * 64 * 64 - 1
    assert call(p(s0), None) == kda.KDA_OK
