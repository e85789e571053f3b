"""Parity of the scalar-gate path (Gated DeltaNet, DeltaNet) through the C ABI
with the fp64 CPU oracle.

Same bar as the per-channel path (max |gpu - oracle| / rms(oracle), outputs and
final states): 2e-3 for bf16 inputs, 1e-5 for fp32 inputs.  The scalar gate of
a workload is channel 0 of its per-channel log_alpha draw: logsigmoid of a
normal, one value per token and head.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_109_b200 as kda
import oracle
from gated_delta_rule_109_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-3, "f32": 1e-5}
NAMES = ("q", "k", "v", "g", "beta")


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gated_delta_rule_109_b200 import build
    build.build()


def _inputs(w, gate="scalar"):
    x = I.make_inputs(w, "cuda")
    x["g"] = x.pop("log_alpha")[..., 0].contiguous() if gate == "scalar" else None
    return x


def _run(x, s0="input", **kw):
    init = x["initial_state"] if s0 == "input" else s0
    out, sT = kda.gdn_forward(x["q"], x["k"], x["v"], x["g"], x["beta"], init, **kw)
    torch.cuda.synchronize()
    kda.check_status()
    return out, sT


def _compare(dtype, x, out, sT, s0="input"):
    init = x["initial_state"] if s0 == "input" else s0
    o_ref, s_ref = oracle.gdn_forward(x["q"], x["k"], x["v"], x["g"], x["beta"], init)
    e_o = oracle.parity_error(out.cpu().numpy(), o_ref)
    assert e_o <= TOL[dtype], "output error %.3g" % e_o
    if sT is not None:
        e_s = oracle.parity_error(sT.cpu().numpy(), s_ref)
        assert e_s <= TOL[dtype], "state error %.3g" % e_s


# ------------------------------------------------------------ shape sweep
SWEEP = []
for gate in ("scalar", "none"):
    for dt in ("bf16", "f32"):
        for d in (64, 128):
            for T in (1, 63, 64, 65, 200):
                SWEEP.append((gate, dt, d, d, T, 2, 3, True))
            SWEEP.append((gate, dt, d, d, 130, 3, 4, False))
SWEEP += [("scalar", "bf16", 128, 64, 100, 2, 3, True), ("scalar", "f32", 64, 128, 100, 2, 3, True)]


# kda_gdn_forward takes the two-kernel prefill on a pooled workspace for bf16 with
# dk = dv = 128; the one-kernel scalar-gate prefill is swept on those shapes too
PATHS = [(case, False) for case in SWEEP]
PATHS += [(case, True) for case in SWEEP if case[1:4] == ("bf16", 128, 128)]


@pytest.mark.parametrize("gate,dt,dk,dv,T,B,H,state,one_kernel", [c + (o,) for c, o in PATHS])
def test_gdn_shape_sweep(gate, dt, dk, dv, T, B, H, state, one_kernel):
    w = I.scaled(I.PREFILL_B4_T16K_STATE if state else I.PREFILL_H16_T4K,
                 B=B, H=H, T=T, dk=dk, dv=dv, dtype=dt, seed=2000 + T + dk)
    x = _inputs(w, gate)
    out, sT = _run(x, one_kernel=one_kernel)
    _compare(dt, x, out, sT)


# ------------------------------------------------------------ workload sizes
def test_gdn_prefill_h16_t4096_all_heads():
    x = _inputs(I.PREFILL_H16_T4K)
    out, sT = _run(x)
    _compare("bf16", x, out, sT)


def test_gdn_long_context_h32_t65536_sampled_heads():
    w = I.PREFILL_H32_T64K
    x = _inputs(w)
    out, sT = _run(x)
    assert torch.isfinite(out).all() and torch.isfinite(sT).all()
    for b, h in [(0, 0), (0, 19)]:
        sub = {n: x[n][b:b + 1, :, h:h + 1].contiguous() for n in NAMES}
        o_ref, s_ref = oracle.gdn_forward(sub["q"], sub["k"], sub["v"], sub["g"], sub["beta"], None)
        assert oracle.parity_error(out[b:b + 1, :, h:h + 1].cpu().numpy(), o_ref) <= TOL["bf16"]
        assert oracle.parity_error(sT[b:b + 1, h:h + 1].cpu().numpy(), s_ref) <= TOL["bf16"]


def test_gdn_matches_kda_with_broadcast_gate():
    """KDA with every channel of log_alpha equal to the scalar gate is Gated DeltaNet."""
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=2, H=4, T=333, seed=17)
    x = _inputs(w)
    out_g, s_g = _run(x)
    la = x["g"][..., None].expand(-1, -1, -1, w.dk).contiguous()
    out_k, s_k = kda.forward(x["q"], x["k"], x["v"], la, x["beta"], x["initial_state"])
    torch.cuda.synchronize()
    assert oracle.parity_error(out_g.cpu().numpy(), out_k.cpu().double().numpy()) <= 2 * TOL["bf16"]
    assert oracle.parity_error(s_g.cpu().numpy(), s_k.cpu().double().numpy()) <= 2 * TOL["bf16"]


# ------------------------------------------------------------ edge values
@pytest.mark.parametrize("dt,one_kernel", [("bf16", False), ("bf16", True), ("f32", False)])
@pytest.mark.parametrize("case", ["decay_minus5", "forget_all_minus100", "tiny_decay", "beta0", "beta1",
                                  "mixed_extreme"])
def test_gdn_extreme_gates(dt, one_kernel, case):
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=1, H=2, T=200, dtype=dt, seed=32)
    x = _inputs(w)
    if case == "decay_minus5":
        x["g"].fill_(-5.0)
    elif case == "forget_all_minus100":
        x["g"].fill_(-100.0)          # e^{G} underflows to 0 inside a chunk
    elif case == "tiny_decay":
        x["g"].fill_(-1e-7)
    elif case == "beta0":
        x["beta"].zero_()
    elif case == "beta1":
        x["beta"].fill_(1.0)
    elif case == "mixed_extreme":
        x["g"][:, 64:128] = -3.0
        x["g"][:, 130:133] = -60.0
    out, sT = _run(x, one_kernel=one_kernel)
    assert torch.isfinite(out).all() and torch.isfinite(sT).all()
    _compare(dt, x, out, sT)


def test_gdn_empty_sequence_and_null_final_state():
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=2, H=3, T=0, seed=6)
    x = _inputs(w)
    fs = torch.full_like(x["initial_state"], float("nan"))
    out, sT = kda.gdn_forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"], final_state=fs)
    torch.cuda.synchronize()
    assert out.numel() == 0 and torch.equal(sT, x["initial_state"])
    w = I.scaled(w, T=90)
    x = _inputs(w, "none")
    out_a, none = _run(x, return_final_state=False)
    assert none is None
    carry = x["initial_state"].clone()
    out_b, _ = _run(x, s0=carry, final_state=carry)
    assert torch.equal(out_a, out_b)
    _compare("bf16", x, out_b, carry)


# ------------------------------------------------------------ decode
@pytest.mark.parametrize("gate", ["scalar", "none"])
@pytest.mark.parametrize("dt,d", [("bf16", 128), ("f32", 64)])
def test_gdn_decode_steps_reproduce_prefill(gate, dt, d):
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=3, H=4, T=70, dk=d, dv=d, dtype=dt, seed=42)
    x = _inputs(w, gate)
    out_p, sT_p = _run(x)
    state = x["initial_state"].clone()
    outs = []
    for t in range(w.T):
        g = None if x["g"] is None else x["g"][:, t].contiguous()
        outs.append(kda.gdn_decode_step(x["q"][:, t].contiguous(), x["k"][:, t].contiguous(),
                                        x["v"][:, t].contiguous(), g, x["beta"][:, t].contiguous(), state))
    torch.cuda.synchronize()
    out_d = torch.stack(outs, dim=1)
    _compare(dt, x, out_d, state)
    assert oracle.parity_error(out_d.cpu().numpy(), out_p.cpu().double().numpy()) <= 2 * TOL[dt]
    assert oracle.parity_error(state.cpu().numpy(), sT_p.cpu().double().numpy()) <= 2 * TOL[dt]


# ------------------------------------------------------------ memory safety and determinism
def test_gdn_outputs_fully_written_and_guards_untouched():
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=3, H=5, T=131, seed=56)
    x = _inputs(w)
    n_out, n_st, G = w.B * w.T * w.H * w.dv, w.B * w.H * w.dk * w.dv, 4096
    ob = torch.full((G + n_out + G,), float("nan"), device="cuda")
    sb = torch.full((G + n_st + G,), float("nan"), device="cuda")
    out = ob[G:G + n_out].view(w.B, w.T, w.H, w.dv)
    sT = sb[G:G + n_st].view(w.B, w.H, w.dk, w.dv)
    _run(x, out=out, final_state=sT)
    assert torch.isfinite(out).all() and torch.isfinite(sT).all()
    assert torch.isnan(ob[:G]).all() and torch.isnan(ob[G + n_out:]).all()
    assert torch.isnan(sb[:G]).all() and torch.isnan(sb[G + n_st:]).all()


def test_gdn_deterministic():
    x = _inputs(I.scaled(I.PREFILL_H16_T4K, H=4, T=1000, seed=67))
    o1, s1 = _run(x)
    o2, s2 = _run(x)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_gdn_binding_rejects_per_channel_gate():
    x = I.make_inputs(I.scaled(I.PREFILL_H16_T4K, H=2, T=10), "cuda")
    with pytest.raises(ValueError):
        kda.gdn_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"])


# ------------------------------------------------------------ two-kernel path with a workspace
@pytest.mark.parametrize("gate,T,B,H,state", [("scalar", 1, 1, 2, True), ("scalar", 65, 2, 3, True),
                                              ("scalar", 200, 1, 4, False), ("none", 130, 2, 2, True),
                                              ("scalar", 333, 2, 20, True), ("none", 64, 1, 40, False)])
def test_gdn_workspace_path(gate, T, B, H, state):
    """kda_gdn_forward_ws: the scalar decay (or none) staged in every key channel of
    the two-kernel prefill; slice and full-head chain kernels both covered."""
    w = I.scaled(I.PREFILL_B4_T16K_STATE if state else I.PREFILL_H16_T4K, B=B, H=H, T=T, seed=9000 + T + H)
    x = _inputs(w, gate)
    ws = kda.make_workspace(w.B, w.T, w.H, 128, 128)
    out, sT = _run(x, workspace=ws)
    _compare("bf16", x, out, sT)


def test_gdn_persistent_chunk_local_kernel_many_chunks_per_cta():
    """More chunks than two per SM, so each CTA of the persistent scalar-gate kernel
    walks several, loading the next one's inputs while it finishes the current: a
    ragged last chunk (4 tokens), a wide-range chunk among them, a carried state;
    blocked workspaces give the same bits."""
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=1, H=8, T=4100, seed=9150)
    assert w.B * w.H * ((w.T + 63) // 64) > 2 * torch.cuda.get_device_properties(0).multi_processor_count
    x = _inputs(w)
    x["g"][:, 640:704] = -4.0         # range 256 in that chunk: factors pair by pair
    ws_full = kda.make_workspace(w.B, w.T, w.H, 128, 128)
    out_f, s_f = _run(x, workspace=ws_full)
    _compare("bf16", x, out_f, s_f)
    bh, rec = w.B * w.H, kda.workspace_bytes(1, 64, 1, 128, 128)
    ws_b = kda.make_workspace(w.B, w.T, w.H, 128, 128, nbytes=bh * rec * 7 + bh * 128 * 128 * 4)
    out_b, s_b = _run(x, workspace=ws_b)
    assert torch.equal(out_f, out_b) and torch.equal(s_f, s_b)


def test_gdn_workspace_path_strong_decay_and_blocks():
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=1, H=3, T=300, seed=9100)
    x = _inputs(w)
    x["g"][:, 64:128] = -3.0          # range 192 per chunk: the wide-range (pairwise) path
    ws_full = kda.make_workspace(w.B, w.T, w.H, 128, 128)
    out_f, s_f = _run(x, workspace=ws_full)
    _compare("bf16", x, out_f, s_f)
    bh, rec = w.B * w.H, kda.workspace_bytes(1, 64, 1, 128, 128)
    ws_b = kda.make_workspace(w.B, w.T, w.H, 128, 128, nbytes=bh * rec * 2 + bh * 128 * 128 * 4)
    out_b, s_b = _run(x, workspace=ws_b)
    assert torch.equal(out_f, out_b) and torch.equal(s_f, s_b)


def test_gdn_workspace_long_context_sampled_heads():
    w = I.PREFILL_H32_T64K
    x = _inputs(w)
    ws = kda.make_workspace(w.B, w.T, w.H, 128, 128)
    out, sT = _run(x, workspace=ws)
    for h in (0, 19):
        sub = {n: x[n][:, :, h:h + 1].contiguous() for n in ("q", "k", "v", "g", "beta")}
        o_ref, s_ref = oracle.gdn_forward(sub["q"], sub["k"], sub["v"], sub["g"], sub["beta"], None)
        assert oracle.parity_error(out[:, :, h:h + 1].cpu().numpy(), o_ref) <= TOL["bf16"]
        assert oracle.parity_error(sT[:, h:h + 1].cpu().numpy(), s_ref) <= TOL["bf16"]
