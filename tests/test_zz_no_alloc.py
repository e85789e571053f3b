"""kda_forward_noalloc: the two-kernel prefill on the library's own scratch.

The call takes no workspace and allocates nothing; its scratch is a fixed array
in the library's device image.  Checked here: parity with the fp64 oracle,
bit-identity with kda_forward_ws given a workspace of the same size, no device
memory growth, ordering of calls on different streams, the fallback for other
dtypes, and argument checks before anything touches CUDA.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_109_b200 as kda
import oracle
from gated_delta_rule_109_b200 import inputs as I

TOL = 2e-3
NAMES = ("q", "k", "v", "log_alpha", "beta")
FAKE = 0x100000


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_109_b200 import build
    build.build()
    return kda.load()


# ------------------------------------------------------------ host side (no GPU)
def test_scratch_size_and_argument_checks(lib):
    assert kda.noalloc_scratch_bytes() == 128 << 20

    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, s0=None, out=FAKE, sT=None, B=1, T=8, H=2)
        a.update(kw)
        return lib.kda_forward_noalloc(a["q"], a["k"], a["v"], a["la"], a["beta"], a["s0"], a["out"], a["sT"],
                                       a["B"], a["T"], a["H"], 128, 128, kda.KDA_BF16, ctypes.c_float(0.0), None)
    assert call(q=None) == kda.KDA_ERR_INVALID_ARG
    assert call(B=0) == kda.KDA_ERR_INVALID_ARG
    assert call(la=FAKE + 4) == kda.KDA_ERR_MISALIGNED
    assert call(sT=FAKE + 8) == kda.KDA_ERR_MISALIGNED


# ------------------------------------------------------------ GPU
gpu = pytest.mark.gpu


def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _compare(x, out, sT):
    o_ref, s_ref = oracle.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["initial_state"])
    assert oracle.parity_error(out.cpu().numpy(), o_ref) <= TOL
    assert oracle.parity_error(sT.cpu().numpy(), s_ref) <= TOL


@gpu
@pytest.mark.parametrize("B,H,T,state", [(1, 4, 1000, True), (2, 3, 65, False), (2, 20, 200, True)])
def test_noalloc_parity(lib, B, H, T, state):
    _cuda()
    w = I.scaled(I.PREFILL_B4_T16K_STATE if state else I.PREFILL_H16_T4K, B=B, H=H, T=T, seed=5000 + T)
    x = I.make_inputs(w, "cuda")
    out, sT = kda.forward_noalloc(*(x[n] for n in NAMES), x["initial_state"])
    torch.cuda.synchronize()
    kda.check_status()
    _compare(x, out, sT)


@gpu
def test_noalloc_long_context_matches_equal_workspace(lib):
    """B1 H32 T65536 does not fit the scratch whole: it runs in blocks, bit-identical
    to kda_forward_ws with a workspace of the scratch's size."""
    _cuda()
    w = I.PREFILL_H32_T64K
    x = I.make_inputs(w, "cuda")
    args = [x[n] for n in NAMES]
    out_n, s_n = kda.forward_noalloc(*args, None)
    ws = torch.empty(kda.noalloc_scratch_bytes(), dtype=torch.uint8, device="cuda")
    assert kda.workspace_bytes(w.B, w.T, w.H, 128, 128) > ws.numel()
    out_w, s_w = kda.forward(*args, None, workspace=ws)
    torch.cuda.synchronize()
    kda.check_status()
    assert torch.equal(out_n, out_w) and torch.equal(s_n, s_w)
    for h in (0, 21):
        sub = {n: x[n][:, :, h:h + 1].contiguous() for n in NAMES}
        o_ref, s_ref = oracle.forward(sub["q"], sub["k"], sub["v"], sub["log_alpha"], sub["beta"], None)
        assert oracle.parity_error(out_n[:, :, h:h + 1].cpu().numpy(), o_ref) <= TOL
        assert oracle.parity_error(s_n[:, h:h + 1].cpu().numpy(), s_ref) <= TOL


@gpu
def test_noalloc_allocates_nothing(lib):
    _cuda()
    w = I.scaled(I.PREFILL_H16_T4K, H=8, T=8192, seed=51)
    x = I.make_inputs(w, "cuda")
    out = torch.empty((1, w.T, w.H, 128), device="cuda")
    sT = torch.empty((1, w.H, 128, 128), device="cuda")
    kda.forward_noalloc(*(x[n] for n in NAMES), None, out=out, final_state=sT)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        kda.forward_noalloc(*(x[n] for n in NAMES), None, out=out, final_state=sT)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0


@gpu
def test_noalloc_calls_on_two_streams_are_ordered(lib):
    """Two streams share the scratch; the library orders their calls."""
    _cuda()
    ws_ = [I.scaled(I.PREFILL_B4_T16K_STATE, B=2, H=8, T=3000, seed=s) for s in (61, 62)]
    xs = [I.make_inputs(w, "cuda") for w in ws_]
    refs = []
    for x in xs:
        refs.append(kda.forward_noalloc(*(x[n] for n in NAMES), x["initial_state"]))
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    results = [None, None]
    for rep in range(3):
        for i, (st, x) in enumerate(zip(streams, xs)):
            with torch.cuda.stream(st):
                results[i] = kda.forward_noalloc(*(x[n] for n in NAMES), x["initial_state"])
    torch.cuda.synchronize()
    kda.check_status()
    for (o, s), (ro, rs) in zip(results, refs):
        assert torch.equal(o, ro) and torch.equal(s, rs)


@gpu
def test_noalloc_other_shapes_are_kda_forward(lib):
    _cuda()
    w = I.scaled(I.TINY_F32, T=130, seed=71)
    x = I.make_inputs(w, "cuda")
    out_n, s_n = kda.forward_noalloc(*(x[n] for n in NAMES), None)
    out_f, s_f = kda.forward(*(x[n] for n in NAMES), None)
    torch.cuda.synchronize()
    assert torch.equal(out_n, out_f) and torch.equal(s_n, s_f)
