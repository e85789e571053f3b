"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Bar (max |gpu - oracle| / rms(oracle), for outputs and final states):
2e-3 for bf16 inputs, 1e-5 for fp32 inputs.
"""
import math

import numpy as np
import pytest
import torch

import gated_delta_rule_109_b200 as kda
import oracle
from gated_delta_rule_109_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-3, "f32": 1e-5}


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gated_delta_rule_109_b200 import build
    build.build()


def _run_gpu(x, with_state_out=True, initial_state="input", one_kernel=False):
    s0 = x["initial_state"] if initial_state == "input" else initial_state
    out, sT = kda.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], s0,
                          return_final_state=with_state_out, one_kernel=one_kernel)
    torch.cuda.synchronize()
    kda.check_status()
    return out, sT


def _compare(w, x, out, sT, s0="input", tol=None):
    tol = TOL[w.dtype] if tol is None else tol
    init = x["initial_state"] if s0 == "input" else s0
    o_ref, s_ref = oracle.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], init)
    e_o = oracle.parity_error(out.cpu().numpy(), o_ref)
    assert e_o <= tol, "output error %.3g > %.3g" % (e_o, tol)
    if sT is not None:
        e_s = oracle.parity_error(sT.cpu().numpy(), s_ref)
        assert e_s <= tol, "state error %.3g > %.3g" % (e_s, tol)
    return e_o


# ------------------------------------------------------------ the named workloads
def test_tiny_f32_workload():
    w = I.TINY_F32
    x = I.make_inputs(w, "cuda")
    out, sT = _run_gpu(x)
    _compare(w, x, out, sT)


def test_prefill_h16_t4096_workload():
    w = I.PREFILL_H16_T4K
    x = I.make_inputs(w, "cuda")
    out, sT = _run_gpu(x)
    _compare(w, x, out, sT)


def _sampled_heads(w, x, out, sT, pairs):
    """Compare full-length outputs and final states of some (b, h) pairs."""
    for b, h in pairs:
        sub = {n: x[n][b:b + 1, :, h:h + 1].contiguous() for n in ("q", "k", "v", "log_alpha", "beta")}
        s0 = None if x["initial_state"] is None else x["initial_state"][b:b + 1, h:h + 1].contiguous()
        o_ref, s_ref = oracle.forward(sub["q"], sub["k"], sub["v"], sub["log_alpha"], sub["beta"], s0)
        e_o = oracle.parity_error(out[b:b + 1, :, h:h + 1].cpu().numpy(), o_ref)
        e_s = oracle.parity_error(sT[b:b + 1, h:h + 1].cpu().numpy(), s_ref)
        assert e_o <= TOL[w.dtype] and e_s <= TOL[w.dtype], (b, h, e_o, e_s)


def test_long_context_h32_t65536_sampled_heads():
    w = I.PREFILL_H32_T64K
    x = I.make_inputs(w, "cuda")
    out, sT = _run_gpu(x)
    assert torch.isfinite(out).all() and torch.isfinite(sT).all()
    _sampled_heads(w, x, out, sT, [(0, 0), (0, 13), (0, 31)])


def test_batched_carried_state_b4_t16384_sampled_heads():
    w = I.PREFILL_B4_T16K_STATE
    x = I.make_inputs(w, "cuda")
    out, sT = _run_gpu(x)
    assert torch.isfinite(out).all() and torch.isfinite(sT).all()
    _sampled_heads(w, x, out, sT, [(0, 0), (1, 7), (2, 20), (3, 31)])


def test_decode_b256_h32_all_heads_two_steps():
    w = I.DECODE_B256
    x = I.make_inputs(w, "cuda", steps=2)
    state = x["initial_state"].clone()
    ref_state = x["initial_state"].cpu().double().numpy()
    for s in range(2):
        o = kda.decode_step(x["q"][s], x["k"][s], x["v"][s], x["log_alpha"][s], x["beta"][s], state)
        torch.cuda.synchronize()
        ins = {n: x[n][s].unsqueeze(1) for n in ("q", "k", "v", "log_alpha", "beta")}
        o_ref, ref_state = oracle.forward(ins["q"], ins["k"], ins["v"], ins["log_alpha"], ins["beta"], ref_state)
        assert oracle.parity_error(o.cpu().numpy(), o_ref[:, 0]) <= TOL["bf16"]
        assert oracle.parity_error(state.cpu().numpy(), ref_state) <= TOL["bf16"]


# ------------------------------------------------------------ shape sweep
SWEEP = []
for dt in ("bf16", "f32"):
    for d in (64, 128):
        for T in (1, 15, 63, 64, 65, 127, 200):
            SWEEP.append((dt, d, d, T, 1, 1, True))
        SWEEP.append((dt, d, d, 130, 3, 4, True))
        SWEEP.append((dt, d, d, 130, 3, 4, False))
SWEEP += [("bf16", 128, 64, 100, 2, 3, True), ("f32", 64, 128, 100, 2, 3, True)]


# kda_forward takes the two-kernel prefill on a pooled workspace for bf16 with
# dk = dv = 128; the one-kernel prefill (no workspace) is swept on those shapes too
PATHS = [(case, False) for case in SWEEP]
PATHS += [(case, True) for case in SWEEP if case[:3] == ("bf16", 128, 128)]


@pytest.mark.parametrize("dt,dk,dv,T,B,H,state,one_kernel", [c + (o,) for c, o in PATHS])
def test_shape_sweep(dt, dk, dv, T, B, H, state, one_kernel):
    w = I.scaled(I.PREFILL_B4_T16K_STATE if state else I.PREFILL_H16_T4K,
                 B=B, H=H, T=T, dk=dk, dv=dv, dtype=dt, seed=1000 + T + dk)
    x = I.make_inputs(w, "cuda")
    out, sT = _run_gpu(x, one_kernel=one_kernel)
    _compare(w, x, out, sT)


def test_null_final_state_and_aliasing():
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=2, H=3, T=150, seed=77)
    x = I.make_inputs(w, "cuda")
    out_a, none = _run_gpu(x, with_state_out=False)
    assert none is None
    # final_state aliasing initial_state: in-place carry
    carry = x["initial_state"].clone()
    out_b, sT = kda.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], carry, final_state=carry)
    torch.cuda.synchronize()
    assert sT.data_ptr() == carry.data_ptr()
    assert torch.equal(out_a, out_b)
    _compare(w, x, out_b, carry)


def test_empty_sequence_copies_or_zeroes_state():
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=2, H=3, T=0, seed=5)
    x = I.make_inputs(w, "cuda")
    fs = torch.full_like(x["initial_state"], float("nan"))
    out, sT = kda.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["initial_state"], final_state=fs)
    torch.cuda.synchronize()
    assert out.numel() == 0 and torch.equal(sT, x["initial_state"])
    out, sT = kda.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], None, final_state=fs)
    torch.cuda.synchronize()
    assert torch.count_nonzero(sT) == 0


def test_split_sequence_carry_matches_single_pass():
    """Prefill of T tokens == prefill of T1 then T - T1 with the state carried (chunk tails)."""
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=1, H=2, T=300, seed=9)
    x = I.make_inputs(w, "cuda")
    out, sT = _run_gpu(x)
    T1 = 77
    a = {n: x[n][:, :T1].contiguous() for n in ("q", "k", "v", "log_alpha", "beta")}
    b = {n: x[n][:, T1:].contiguous() for n in ("q", "k", "v", "log_alpha", "beta")}
    o1, s1 = kda.forward(a["q"], a["k"], a["v"], a["log_alpha"], a["beta"], x["initial_state"])
    o2, s2 = kda.forward(b["q"], b["k"], b["v"], b["log_alpha"], b["beta"], s1)
    torch.cuda.synchronize()
    ref = np.concatenate([o1.cpu().numpy(), o2.cpu().numpy()], axis=1)
    assert oracle.parity_error(ref, out.cpu().numpy()) <= TOL["bf16"]
    assert oracle.parity_error(s2.cpu().numpy(), sT.cpu().numpy()) <= TOL["bf16"]


# ------------------------------------------------------------ edge values
@pytest.mark.parametrize("dt,one_kernel", [("bf16", False), ("bf16", True), ("f32", False)])
@pytest.mark.parametrize("case", ["decay_minus5", "near_threshold", "no_decay", "beta0", "beta1",
                                  "mixed_extreme"])
def test_extreme_gates(dt, one_kernel, case):
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=1, H=2, T=200, dtype=dt, seed=31)
    x = I.make_inputs(w, "cuda")
    if case == "decay_minus5":
        x["log_alpha"].fill_(-5.0)
    elif case == "near_threshold":
        # a log-decay range of 76.8 per chunk: the split exponentials reach exp(+-38.4)
        x["log_alpha"].fill_(-1.2)
    elif case == "no_decay":
        x["log_alpha"].zero_()
    elif case == "beta0":
        x["beta"].zero_()
    elif case == "beta1":
        x["beta"].fill_(1.0)
    elif case == "mixed_extreme":
        # one chunk of very strong forgetting in the middle of mild ones
        x["log_alpha"][:, 64:128] = -3.0
        x["log_alpha"][:, 128:140, :, :7] = -20.0
    out, sT = _run_gpu(x, one_kernel=one_kernel)
    assert torch.isfinite(out).all() and torch.isfinite(sT).all()
    _compare(w, x, out, sT)


# ------------------------------------------------------------ decode
@pytest.mark.parametrize("dt,d", [("bf16", 128), ("bf16", 64), ("f32", 128), ("f32", 64)])
def test_decode_steps_reproduce_prefill(dt, d):
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=3, H=4, T=70, dk=d, dv=d, dtype=dt, seed=41)
    x = I.make_inputs(w, "cuda")
    out_p, sT_p = _run_gpu(x)
    state = x["initial_state"].clone()
    outs = []
    for t in range(w.T):
        outs.append(kda.decode_step(x["q"][:, t].contiguous(), x["k"][:, t].contiguous(),
                                    x["v"][:, t].contiguous(), x["log_alpha"][:, t].contiguous(),
                                    x["beta"][:, t].contiguous(), state))
    torch.cuda.synchronize()
    out_d = torch.stack(outs, dim=1)
    _compare(w, x, out_d, state)
    tol = TOL[dt]
    assert oracle.parity_error(out_d.cpu().numpy(), out_p.cpu().double().numpy()) <= 2 * tol
    assert oracle.parity_error(state.cpu().numpy(), sT_p.cpu().double().numpy()) <= 2 * tol


# ------------------------------------------------------------ memory safety and determinism
def test_outputs_fully_written_and_guards_untouched():
    """NaN-poisoned outputs must be fully overwritten; guard regions around them unchanged."""
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=3, H=5, T=131, seed=55)
    x = I.make_inputs(w, "cuda")
    n_out = w.B * w.T * w.H * w.dv
    n_st = w.B * w.H * w.dk * w.dv
    G = 4096
    ob = torch.full((G + n_out + G,), float("nan"), device="cuda")
    sb = torch.full((G + n_st + G,), float("nan"), device="cuda")
    out = ob[G:G + n_out].view(w.B, w.T, w.H, w.dv)
    sT = sb[G:G + n_st].view(w.B, w.H, w.dk, w.dv)
    kda.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["initial_state"], out=out, final_state=sT)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all() and torch.isfinite(sT).all()
    assert torch.isnan(ob[:G]).all() and torch.isnan(ob[G + n_out:]).all()
    assert torch.isnan(sb[:G]).all() and torch.isnan(sb[G + n_st:]).all()
    # decode, same check
    st = x["initial_state"].clone()
    db = torch.full((G + w.B * w.H * w.dv + G,), float("nan"), device="cuda")
    o = db[G:G + w.B * w.H * w.dv].view(w.B, w.H, w.dv)
    kda.decode_step(x["q"][:, 0].contiguous(), x["k"][:, 0].contiguous(), x["v"][:, 0].contiguous(),
                    x["log_alpha"][:, 0].contiguous(), x["beta"][:, 0].contiguous(), st, out=o)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and torch.isnan(db[:G]).all() and torch.isnan(db[G + o.numel():]).all()


def test_deterministic():
    w = I.scaled(I.PREFILL_H16_T4K, B=1, H=4, T=1000, seed=66)
    x = I.make_inputs(w, "cuda")
    o1, s1 = _run_gpu(x)
    o2, s2 = _run_gpu(x)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_no_device_memory_grows_with_sequence_length():
    """Device memory does not grow with T (the fixed-state property measured on the
    first page's demo): the one-kernel prefill takes nothing, and kda_forward's
    pooled workspace is two blocks of 64 chunks once the sequence is long enough,
    whatever T; a repeated call of a shape takes no new memory."""
    kda.workspace_pool_trim()
    assert kda.workspace_pool_bytes() == 0
    for T in (4096, 16384, 65536):
        w = I.scaled(I.PREFILL_H16_T4K, H=4, T=T, seed=3)
        x = I.make_inputs(w, "cuda")
        out = torch.empty((1, T, 4, 128), device="cuda")
        sT = torch.empty((1, 4, 128, 128), device="cuda")
        for one_kernel in (True, False):
            kda.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], None, out=out, final_state=sT,
                        one_kernel=one_kernel)
            torch.cuda.synchronize()
            free0 = torch.cuda.mem_get_info()[0]
            kda.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], None, out=out, final_state=sT,
                        one_kernel=one_kernel)
            torch.cuda.synchronize()
            assert torch.cuda.mem_get_info()[0] == free0, (T, one_kernel)
    # pipelined sizes do not depend on T; the pool holds the two shapes' workspaces
    ws_long = kda.workspace_bytes(1, 65536, 4, 128, 128)
    assert ws_long == kda.workspace_bytes(1, 16384, 4, 128, 128)
    held = kda.workspace_pool_bytes()
    assert ws_long <= held <= kda.workspace_bytes(1, 4096, 4, 128, 128) + ws_long + (64 << 20)
    free_before = torch.cuda.mem_get_info()[0]
    kda.workspace_pool_trim()
    assert kda.workspace_pool_bytes() == 0
    assert torch.cuda.mem_get_info()[0] >= free_before + held // 2


def test_pooled_workspace_falls_back_to_the_one_kernel_prefill():
    """A shape whose smallest workspace cannot be had (1.5 M heads of one token: 223 GB
    of records) runs the one-kernel prefill, bit for bit; the pool keeps no more than its
    1 GiB (the failed request may leave memory it reserved on the way, up to that bound)
    and the CUDA error state is clean."""
    w = I.scaled(I.PREFILL_H16_T4K, B=1, H=1_500_000, T=1, seed=21)
    assert kda.workspace_bytes(w.B, w.T, w.H, 128, 128, minimum=True) > torch.cuda.get_device_properties(0).total_memory
    x = I.make_inputs(w, "cuda")
    args = (x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], None)
    held = kda.workspace_pool_bytes()
    out_p, _ = kda.forward(*args, return_final_state=False)
    out_1, _ = kda.forward(*args, return_final_state=False, one_kernel=True)
    torch.cuda.synchronize()
    kda.check_status()
    assert torch.equal(out_p, out_1)
    assert kda.workspace_pool_bytes() <= max(held, 1 << 30) + (64 << 20)
    kda.workspace_pool_trim()
    assert kda.workspace_pool_bytes() == 0
    # and the library still takes the pooled path for an ordinary shape afterwards
    wb = I.scaled(I.PREFILL_B4_T16K_STATE, B=1, H=2, T=200, seed=22)
    xb = I.make_inputs(wb, "cuda")
    ws = kda.make_workspace(wb.B, wb.T, wb.H, 128, 128)
    o_w, s_w = kda.forward(xb["q"], xb["k"], xb["v"], xb["log_alpha"], xb["beta"], xb["initial_state"], workspace=ws)
    o_p, s_p = _run_gpu(xb)
    assert torch.equal(o_p, o_w) and torch.equal(s_p, s_w)


def test_pooled_workspace_is_capped_and_shared_by_streams():
    """A shape whose fastest workspace is above 1 GiB runs in blocks within 1 GiB
    (bit-identical to the full workspace); calls on two streams take their own
    workspaces from the pool."""
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=4, H=32, T=8192, seed=13)
    assert kda.workspace_bytes(w.B, w.T, w.H, 128, 128) > (1 << 30)
    x = I.make_inputs(w, "cuda")
    ws = kda.make_workspace(w.B, w.T, w.H, 128, 128)
    o_ws, s_ws = kda.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["initial_state"], workspace=ws)
    del ws
    kda.workspace_pool_trim()
    o_p, s_p = _run_gpu(x)
    assert torch.equal(o_p, o_ws) and torch.equal(s_p, s_ws)
    assert kda.workspace_pool_bytes() <= (1 << 30) + (64 << 20)
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    res = [None, None]
    for i, st in enumerate(streams):
        with torch.cuda.stream(st):
            res[i] = kda.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["initial_state"])
    torch.cuda.synchronize()
    kda.check_status()
    for o, s in res:
        assert torch.equal(o, o_ws) and torch.equal(s, s_ws)


def test_binding_rejects_mismatched_tensors():
    w = I.scaled(I.PREFILL_H16_T4K, H=2, T=10)
    x = I.make_inputs(w, "cuda")
    with pytest.raises(TypeError):
        kda.forward(x["q"], x["k"].float(), x["v"], x["log_alpha"], x["beta"])
    with pytest.raises(ValueError):
        kda.forward(x["q"], x["k"], x["v"], x["log_alpha"][:, :5], x["beta"])
    with pytest.raises(kda.KDAError):
        kda.forward(x["q"][..., :96].contiguous(), x["k"][..., :96].contiguous(), x["v"],
                    x["log_alpha"][..., :96].contiguous(), x["beta"])
