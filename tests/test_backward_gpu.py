"""Parity of kda_backward (the gradients of the forward) with the fp64 oracle.

The oracle differentiates the token recurrence with torch.autograd in fp64
(oracle.backward, pinned by finite differences and a closed form).  The CUDA
path computes in fp32; the bar, max |gpu - oracle| / rms(oracle) per gradient,
is 1e-4: fp32 rounding (unit roundoff 6e-8) accumulated along a recurrence of
up to 4096 tokens, with a margin of about two.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_109_b200 as kda
import oracle
from gated_delta_rule_109_b200 import inputs as I

pytestmark = pytest.mark.gpu
TOL = 1e-4
NAMES = ("q", "k", "v", "log_alpha", "beta")
GRADS = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dinitial_state")


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gated_delta_rule_109_b200 import build
    build.build()


def _cotangents(w, seed, final=True):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    d_out = torch.randn((w.B, w.T, w.H, w.dv), generator=g, device="cuda")
    d_fin = torch.randn((w.B, w.H, w.dk, w.dv), generator=g, device="cuda") if final else None
    return d_out, d_fin


def _check(x, got, d_out, d_fin, heads=None):
    sel = (lambda a, ax: a) if heads is None else (lambda a, ax: a.narrow(ax, heads[0], heads[1]))
    sub = {n: sel(x[n], 2).contiguous() for n in NAMES}
    s0 = None if x["initial_state"] is None else sel(x["initial_state"], 1).contiguous()
    dfin = None if d_fin is None else sel(d_fin, 1).contiguous()
    ref = oracle.backward(*(sub[n] for n in NAMES), sel(d_out, 2).contiguous(), s0, dfin)
    errs = {}
    for n in GRADS:
        ax = 1 if n == "dinitial_state" else 2
        g = sel(got[n], ax).cpu().numpy()
        errs[n] = oracle.parity_error(g, ref[n])
    assert all(e <= TOL for e in errs.values()), errs
    return errs


SWEEP = [(1, 1, 1, 128, "bf16", True), (15, 1, 2, 128, "bf16", True), (64, 2, 1, 128, "bf16", False),
         (65, 1, 2, 128, "bf16", True), (130, 2, 2, 128, "bf16", True), (200, 1, 3, 64, "bf16", True),
         (131, 1, 2, 64, "f32", True), (100, 2, 1, 128, "f32", False)]


@pytest.mark.parametrize("T,B,H,d,dt,state", SWEEP)
def test_backward_parity_sweep(T, B, H, d, dt, state):
    w = I.scaled(I.PREFILL_B4_T16K_STATE if state else I.PREFILL_H16_T4K, B=B, H=H, T=T, dk=d, dv=d, dtype=dt,
                 seed=8000 + T + d)
    x = I.make_inputs(w, "cuda")
    d_out, d_fin = _cotangents(w, 8100 + T, final=state)
    got = kda.backward(*(x[n] for n in NAMES), d_out, x["initial_state"], d_fin)
    torch.cuda.synchronize()
    _check(x, got, d_out, d_fin)


def test_backward_strong_decay_and_extreme_beta():
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=1, H=2, T=150, seed=8200)
    x = I.make_inputs(w, "cuda")
    x["log_alpha"][:, 20:40] = -4.0
    x["log_alpha"][:, 60:70, :, :9] = -30.0
    x["beta"][:, 80:90] = 1.0
    x["beta"][:, 90:95] = 0.0
    d_out, d_fin = _cotangents(w, 8201)
    got = kda.backward(*(x[n] for n in NAMES), d_out, x["initial_state"], d_fin)
    torch.cuda.synchronize()
    _check(x, got, d_out, d_fin)


def test_backward_long_sequence_sampled_heads():
    """B1 H16 T4096 (the short-context prefill workload), two heads against the oracle."""
    w = I.PREFILL_H16_T4K
    x = I.make_inputs(w, "cuda")
    d_out, _ = _cotangents(w, 8300, final=False)
    got = kda.backward(*(x[n] for n in NAMES), d_out, None, None)
    torch.cuda.synchronize()
    for h in (0, 11):
        _check(x, got, d_out, None, heads=(h, 1))


def test_backward_empty_sequence_and_no_initial_grad():
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=2, H=3, T=0, seed=8400)
    x = I.make_inputs(w, "cuda")
    d_out, d_fin = _cotangents(w, 8401)
    got = kda.backward(*(x[n] for n in NAMES), d_out, x["initial_state"], d_fin)
    torch.cuda.synchronize()
    assert torch.equal(got["dinitial_state"], d_fin)
    got = kda.backward(*(x[n] for n in NAMES), d_out, x["initial_state"], None)
    torch.cuda.synchronize()
    assert not got["dinitial_state"].any()
    w = I.scaled(w, T=70)
    x = I.make_inputs(w, "cuda")
    d_out, d_fin = _cotangents(w, 8402)
    g1 = kda.backward(*(x[n] for n in NAMES), d_out, x["initial_state"], d_fin, initial_state_grad=False)
    g2 = kda.backward(*(x[n] for n in NAMES), d_out, x["initial_state"], d_fin)
    torch.cuda.synchronize()
    assert g1["dinitial_state"] is None
    assert all(torch.equal(g1[n], g2[n]) for n in GRADS[:5])


def test_backward_deterministic_and_in_bounds():
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=2, H=3, T=131, seed=8500)
    x = I.make_inputs(w, "cuda")
    d_out, d_fin = _cotangents(w, 8501)
    nws = kda.backward_workspace_bytes(w.B, w.T, w.H, 128, 128)
    wsb = torch.full((nws + 4096,), 0x5A, dtype=torch.uint8, device="cuda")
    g1 = kda.backward(*(x[n] for n in NAMES), d_out, x["initial_state"], d_fin, workspace=wsb[:nws])
    g2 = kda.backward(*(x[n] for n in NAMES), d_out, x["initial_state"], d_fin)
    torch.cuda.synchronize()
    assert bool((wsb[nws:] == 0x5A).all())
    for n in GRADS:
        assert torch.equal(g1[n], g2[n]), n
        assert torch.isfinite(g1[n]).all(), n


def test_autograd_function_matches_backward():
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=1, H=2, T=90, seed=8600)
    x = I.make_inputs(w, "cuda")
    leaves = {n: x[n].clone().requires_grad_(True) for n in NAMES}
    s0 = x["initial_state"].clone().requires_grad_(True)
    out, fin = kda.KDAFunction.apply(*(leaves[n] for n in NAMES), s0)
    d_out, d_fin = _cotangents(w, 8601)
    torch.autograd.backward([out, fin], [d_out, d_fin])
    ref = kda.backward(*(x[n] for n in NAMES), d_out, x["initial_state"], d_fin)
    torch.cuda.synchronize()
    for n, key in zip(NAMES, GRADS):
        assert torch.equal(leaves[n].grad.float(), ref[key].to(x[n].dtype).float()), n
    assert torch.equal(s0.grad, ref["dinitial_state"])
