"""Parity of kda_forward_raw (gate activation and q/k normalisation fused into the
two-kernel prefill) with the fp64 oracle's forward_raw, through the C ABI."""
import pytest
import torch

import gated_delta_rule_109_b200 as kda
import oracle
from gated_delta_rule_109_b200 import inputs as I

pytestmark = pytest.mark.gpu
TOL = 2e-3
NAMES = ("q", "k", "v", "gate", "beta")


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gated_delta_rule_109_b200 import build
    build.build()


def _run(x, w, gate_act=True, norm=True, nbytes=None):
    ws = kda.make_workspace(w.B, w.T, w.H, 128, 128, nbytes=nbytes)
    out, sT = kda.forward_raw(*(x[n] for n in NAMES), x["initial_state"], workspace=ws,
                              logsigmoid_gate=gate_act, normalize_qk=norm)
    torch.cuda.synchronize()
    kda.check_status()
    return out, sT


def _compare(x, out, sT, gate_act=True, norm=True):
    o_ref, s_ref = oracle.forward_raw(*(x[n] for n in NAMES), x["initial_state"], logsigmoid_gate=gate_act,
                                      normalize_qk=norm)
    e_o = oracle.parity_error(out.cpu().numpy(), o_ref)
    e_s = oracle.parity_error(sT.cpu().numpy(), s_ref)
    assert e_o <= TOL and e_s <= TOL, (e_o, e_s)


@pytest.mark.parametrize("T,B,H", [(1, 1, 2), (65, 1, 2), (200, 2, 3), (640, 1, 4), (200, 2, 20)])
def test_raw_both_steps(T, B, H):
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=B, H=H, T=T, seed=6000 + T)
    x = I.make_raw_inputs(w, "cuda")
    out, sT = _run(x, w)
    _compare(x, out, sT)


@pytest.mark.parametrize("gate_act,norm", [(True, False), (False, True)])
def test_raw_one_step(gate_act, norm):
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=2, H=3, T=150, seed=6101)
    x = I.make_raw_inputs(w, "cuda")
    if not gate_act:
        x["gate"] = torch.nn.functional.logsigmoid(x["gate"].double()).float()
    if not norm:
        for n in ("q", "k"):
            f = x[n].float()
            x[n] = (f / f.norm(dim=-1, keepdim=True)).to(x[n].dtype)
    out, sT = _run(x, w, gate_act, norm)
    _compare(x, out, sT, gate_act, norm)


def test_raw_wide_range_and_blocked():
    """Very negative gate pre-activations make log alpha ~ x: wide-range chunks take the
    pairwise path, which applies the normalisation too; blocked workspaces agree bit for bit."""
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=1, H=3, T=300, seed=6102)
    x = I.make_raw_inputs(w, "cuda")
    x["gate"][:, 64:128] = -4.0
    x["gate"][:, 140:150, :, :5] = -40.0
    out, sT = _run(x, w)
    _compare(x, out, sT)
    bh, rec = w.B * w.H, kda.workspace_bytes(1, 64, 1, 128, 128)
    out_b, s_b = _run(x, w, nbytes=bh * rec * 2 + bh * 128 * 128 * 4)
    assert torch.equal(out, out_b) and torch.equal(sT, s_b)


def test_raw_matches_preprocessed_inputs():
    """Fused steps == the same steps done first in torch (fp32) and kda_forward_ws."""
    w = I.scaled(I.PREFILL_H16_T4K, H=8, T=2000, seed=6103)
    x = I.make_raw_inputs(w, "cuda")
    out, sT = _run(x, w)
    la = torch.nn.functional.logsigmoid(x["gate"])
    qn = (x["q"].float() / x["q"].float().norm(dim=-1, keepdim=True))
    kn = (x["k"].float() / x["k"].float().norm(dim=-1, keepdim=True))
    ws = kda.make_workspace(w.B, w.T, w.H, 128, 128)
    # the unfused path rounds the normalised rows to bf16; compare at twice the bar
    out_u, s_u = kda.forward(qn.to(torch.bfloat16), kn.to(torch.bfloat16), x["v"], la, x["beta"], None,
                             workspace=ws)
    torch.cuda.synchronize()
    assert oracle.parity_error(out.cpu().numpy(), out_u.cpu().double().numpy()) <= 2 * TOL * 4


def test_raw_rejects_unsupported_and_bad_flags():
    w = I.scaled(I.TINY_F32, T=64, seed=6104)
    x = I.make_raw_inputs(w, "cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(kda.KDAError) as err:
        kda.forward_raw(*(x[n] for n in NAMES), None, workspace=ws)
    assert err.value.status == kda.KDA_ERR_UNSUPPORTED
    lib = kda.load()
    wb = I.scaled(I.PREFILL_H16_T4K, H=2, T=64)
    xb = I.make_raw_inputs(wb, "cuda")
    out = torch.empty((1, 64, 2, 128), device="cuda")
    p = lambda t: t.data_ptr()
    st = lib.kda_forward_raw(p(xb["q"]), p(xb["k"]), p(xb["v"]), p(xb["gate"]), p(xb["beta"]), None, p(out), None,
                             1, 64, 2, 128, 128, kda.KDA_BF16, 0.0, 4, p(ws), ws.numel(), None)
    assert st == kda.KDA_ERR_INVALID_ARG
