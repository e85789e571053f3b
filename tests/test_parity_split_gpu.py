"""Parity of the two-kernel prefill (kda_forward_ws with a workspace) with the
fp64 CPU oracle, through the C ABI.

Same bar as the other prefill paths: max |gpu - oracle| / rms(oracle) <= 2e-3
for outputs and final states (bf16 inputs, dk = dv = 128).
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_109_b200 as kda
import oracle
from gated_delta_rule_109_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL = 2e-3
NAMES = ("q", "k", "v", "log_alpha", "beta")


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gated_delta_rule_109_b200 import build
    build.build()


def _ws(w, nbytes=None):
    ws = kda.make_workspace(w.B, w.T, w.H, w.dk, w.dv, nbytes=nbytes)
    assert ws is not None
    return ws


def _run(x, ws, s0="input", **kw):
    init = x["initial_state"] if s0 == "input" else s0
    out, sT = kda.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], init, workspace=ws, **kw)
    torch.cuda.synchronize()
    kda.check_status()
    return out, sT


def _compare(x, out, sT, s0="input"):
    init = x["initial_state"] if s0 == "input" else s0
    o_ref, s_ref = oracle.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], init)
    e_o = oracle.parity_error(out.cpu().numpy(), o_ref)
    assert e_o <= TOL, "output error %.3g" % e_o
    if sT is not None:
        e_s = oracle.parity_error(sT.cpu().numpy(), s_ref)
        assert e_s <= TOL, "state error %.3g" % e_s


# ------------------------------------------------------------ shape sweep
SWEEP = [(T, 1, 1, True) for T in (1, 15, 63, 64, 65, 127, 200, 640)]
SWEEP += [(130, 3, 4, True), (130, 3, 4, False), (257, 2, 3, True)]


@pytest.mark.parametrize("T,B,H,state", SWEEP)
def test_split_shape_sweep(T, B, H, state):
    w = I.scaled(I.PREFILL_B4_T16K_STATE if state else I.PREFILL_H16_T4K, B=B, H=H, T=T, seed=3000 + T)
    x = I.make_inputs(w, "cuda")
    out, sT = _run(x, _ws(w))
    _compare(x, out, sT)


# ------------------------------------------------------------ one chain CTA per head
# More than SMs / 4 heads (148 SMs: more than 37) take the full-head chain kernel.
@pytest.mark.parametrize("T,B,H,state", [(1, 2, 19, True), (64, 2, 19, True), (200, 2, 19, True),
                                         (131, 1, 40, False), (333, 4, 12, True)])
def test_split_full_head_chain(T, B, H, state):
    assert B * H * 4 > torch.cuda.get_device_properties(0).multi_processor_count
    w = I.scaled(I.PREFILL_B4_T16K_STATE if state else I.PREFILL_H16_T4K, B=B, H=H, T=T, seed=4000 + T)
    x = I.make_inputs(w, "cuda")
    out, sT = _run(x, _ws(w))
    _compare(x, out, sT)


def test_full_head_chain_blocked_and_extreme():
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=2, H=20, T=300, seed=81)
    x = I.make_inputs(w, "cuda")
    x["log_alpha"][:, 64:128] = -3.0
    x["log_alpha"][:, 130:135, :, :9] = -30.0
    out_f, s_f = _run(x, _ws(w))
    bh, rec = w.B * w.H, kda.workspace_bytes(1, 64, 1, 128, 128)
    out_b, s_b = _run(x, _ws(w, bh * rec * 2 + bh * 128 * 128 * 4))
    assert torch.equal(out_f, out_b) and torch.equal(s_f, s_b)
    _compare(x, out_f, s_f)


# ------------------------------------------------------------ blocked workspaces
@pytest.mark.parametrize("blocks", [1, 2, 3, 5])
def test_blocked_workspace_matches_one_block(blocks):
    """A workspace holding fewer chunks runs the sequence in blocks with the state
    carried in the workspace; the arithmetic is the same, so the bits are too."""
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=2, H=3, T=300, seed=77)       # 5 chunks
    x = I.make_inputs(w, "cuda")
    out_full, s_full = _run(x, _ws(w))
    bh, rec = w.B * w.H, kda.workspace_bytes(1, 64, 1, 128, 128)
    nbytes = bh * rec * blocks + bh * 128 * 128 * 4 if blocks < 5 else None
    if blocks == 1:
        assert nbytes == kda.workspace_bytes(w.B, w.T, w.H, 128, 128, minimum=True)
    out_b, s_b = _run(x, _ws(w, nbytes))
    assert torch.equal(out_full, out_b) and torch.equal(s_full, s_b)
    _compare(x, out_b, s_b)


def test_too_small_workspace_takes_the_fused_kernel():
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=1, H=2, T=200, seed=78)
    x = I.make_inputs(w, "cuda")
    small = kda.workspace_bytes(w.B, w.T, w.H, 128, 128, minimum=True) - 256
    out, sT = _run(x, _ws(w, small))
    ref_o, ref_s = _run(x, None, one_kernel=True)
    assert torch.equal(out, ref_o) and torch.equal(sT, ref_s)


# ------------------------------------------------------------ workload sizes
def test_split_prefill_h16_t4096_all_heads():
    w = I.PREFILL_H16_T4K
    x = I.make_inputs(w, "cuda")
    out, sT = _run(x, _ws(w))
    _compare(x, out, sT)


def _sampled_heads(x, out, sT, pairs):
    for b, h in pairs:
        sub = {n: x[n][b:b + 1, :, h:h + 1].contiguous() for n in NAMES}
        s0 = None if x["initial_state"] is None else x["initial_state"][b:b + 1, h:h + 1].contiguous()
        o_ref, s_ref = oracle.forward(sub["q"], sub["k"], sub["v"], sub["log_alpha"], sub["beta"], s0)
        e_o = oracle.parity_error(out[b:b + 1, :, h:h + 1].cpu().numpy(), o_ref)
        e_s = oracle.parity_error(sT[b:b + 1, h:h + 1].cpu().numpy(), s_ref)
        assert e_o <= TOL and e_s <= TOL, (b, h, e_o, e_s)


def test_split_long_context_h32_t65536_sampled_heads():
    w = I.PREFILL_H32_T64K
    x = I.make_inputs(w, "cuda")
    out, sT = _run(x, _ws(w))
    assert torch.isfinite(out).all() and torch.isfinite(sT).all()
    _sampled_heads(x, out, sT, [(0, 0), (0, 17), (0, 31)])


def test_split_batched_carried_state_b4_t16384_sampled_heads():
    w = I.PREFILL_B4_T16K_STATE
    x = I.make_inputs(w, "cuda")
    out, sT = _run(x, _ws(w))
    assert torch.isfinite(out).all() and torch.isfinite(sT).all()
    _sampled_heads(x, out, sT, [(0, 1), (1, 8), (2, 21), (3, 30)])


def test_split_agrees_with_fused_kernel():
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=2, H=4, T=1000, seed=79)
    x = I.make_inputs(w, "cuda")
    out_s, s_s = _run(x, _ws(w))
    out_f, s_f = _run(x, None, one_kernel=True)
    assert oracle.parity_error(out_s.cpu().numpy(), out_f.cpu().double().numpy()) <= 2 * TOL
    assert oracle.parity_error(s_s.cpu().numpy(), s_f.cpu().double().numpy()) <= 2 * TOL


# ------------------------------------------------------------ edge values
@pytest.mark.parametrize("case", ["decay_minus5", "near_threshold", "no_decay", "beta0", "beta1",
                                  "mixed_extreme", "wide_one_channel"])
def test_split_extreme_gates(case):
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=1, H=2, T=200, seed=33)
    x = I.make_inputs(w, "cuda")
    if case == "decay_minus5":
        x["log_alpha"].fill_(-5.0)            # range 320 per chunk: pairwise A and M
    elif case == "near_threshold":
        x["log_alpha"].fill_(-1.2)            # range 76.8: split exponentials up to e^38.4
    elif case == "no_decay":
        x["log_alpha"].zero_()
    elif case == "beta0":
        x["beta"].zero_()
    elif case == "beta1":
        x["beta"].fill_(1.0)
    elif case == "mixed_extreme":
        x["log_alpha"][:, 64:128] = -3.0
        x["log_alpha"][:, 128:140, :, :7] = -20.0
    elif case == "wide_one_channel":
        x["log_alpha"][:, 70:72, :, 5] = -60.0   # one channel of one chunk is wide
    out, sT = _run(x, _ws(w))
    assert torch.isfinite(out).all() and torch.isfinite(sT).all()
    _compare(x, out, sT)


# ------------------------------------------------------------ states, guards, determinism
def test_split_null_final_state_null_initial_and_aliasing():
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=2, H=3, T=150, seed=80)
    x = I.make_inputs(w, "cuda")
    ws = _ws(w)
    out_a, none = _run(x, ws, return_final_state=False)
    assert none is None
    carry = x["initial_state"].clone()
    out_b, sT = _run(x, ws, s0=carry, final_state=carry)
    assert sT.data_ptr() == carry.data_ptr() and torch.equal(out_a, out_b)
    _compare(x, out_b, carry)
    out_c, s_c = _run(x, ws, s0=None)
    _compare(x, out_c, s_c, s0=None)


def test_split_outputs_and_workspace_stay_in_bounds():
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=3, H=5, T=131, seed=57)
    x = I.make_inputs(w, "cuda")
    n_out, n_st, G = w.B * w.T * w.H * w.dv, w.B * w.H * w.dk * w.dv, 4096
    ob = torch.full((G + n_out + G,), float("nan"), device="cuda")
    sb = torch.full((G + n_st + G,), float("nan"), device="cuda")
    out = ob[G:G + n_out].view(w.B, w.T, w.H, w.dv)
    sT = sb[G:G + n_st].view(w.B, w.H, w.dk, w.dv)
    nws = kda.workspace_bytes(w.B, w.T, w.H, 128, 128)
    wsb = torch.full((nws + 8192,), 0xA5, dtype=torch.uint8, device="cuda")
    _run(x, wsb[:nws], out=out, final_state=sT)
    assert torch.isfinite(out).all() and torch.isfinite(sT).all()
    assert torch.isnan(ob[:G]).all() and torch.isnan(ob[G + n_out:]).all()
    assert torch.isnan(sb[:G]).all() and torch.isnan(sb[G + n_st:]).all()
    assert bool((wsb[nws:] == 0xA5).all())
    _compare(x, out, sT)


def test_split_deterministic():
    w = I.scaled(I.PREFILL_H16_T4K, H=4, T=1000, seed=68)
    x = I.make_inputs(w, "cuda")
    ws = _ws(w)
    o1, s1 = _run(x, ws)
    o2, s2 = _run(x, ws)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_split_rejects_misaligned_workspace():
    w = I.scaled(I.PREFILL_H16_T4K, H=2, T=100, seed=69)
    x = I.make_inputs(w, "cuda")
    ws = _ws(w, kda.workspace_bytes(w.B, w.T, w.H, 128, 128) + 256)
    with pytest.raises(kda.KDAError) as err:
        kda.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], workspace=ws[16:])
    assert err.value.status == kda.KDA_ERR_MISALIGNED


# ------------------------------------------------------------ host buffers (kda_forward_host)
@pytest.mark.parametrize("T,B,H,block,state", [(1000, 2, 3, 256, True), (300, 1, 2, 64, False),
                                               (65, 2, 20, 0, True), (4096, 1, 4, 1024, True)])
def test_forward_host_equals_device_path(T, B, H, block, state):
    """Copies and kernels overlapped per block; chunk boundaries are the whole
    sequence's, so the result is the workspace path's, bit for bit."""
    w = I.scaled(I.PREFILL_B4_T16K_STATE if state else I.PREFILL_H16_T4K, B=B, H=H, T=T, seed=9600 + T)
    x = I.make_inputs(w, "cuda")
    out_d, s_d = _run(x, _ws(w))
    host = {n: x[n].cpu().pin_memory() for n in NAMES}
    s0 = x["initial_state"].cpu().pin_memory() if x["initial_state"] is not None else None
    out_h, s_h = kda.forward_host(*(host[n] for n in NAMES), s0, block_tokens=block)
    kda.check_status()
    assert torch.equal(out_h, out_d.cpu()) and torch.equal(s_h, s_d.cpu())


def test_forward_host_pageable_and_f32_and_empty():
    w = I.scaled(I.TINY_F32, T=200, seed=9700)              # fp32 inputs: the SIMT path per block
    x = I.make_inputs(w, "cuda")
    out_d, s_d = _run(x, None)
    host = {n: x[n].cpu() for n in NAMES}                   # pageable host memory
    out_h, s_h = kda.forward_host(*(host[n] for n in NAMES), None, block_tokens=128)
    kda.check_status()
    o_ref, s_ref = oracle.forward(*(host[n] for n in NAMES), None)
    assert oracle.parity_error(out_h.numpy(), o_ref) <= 1e-5 and oracle.parity_error(s_h.numpy(), s_ref) <= 1e-5
    w0 = I.scaled(I.PREFILL_B4_T16K_STATE, B=1, H=2, T=0, seed=9701)
    x0 = I.make_inputs(w0, "cpu")
    out0, s0 = kda.forward_host(*(x0[n] for n in NAMES), x0["initial_state"])
    assert out0.numel() == 0 and torch.equal(s0, x0["initial_state"])


# ------------------------------------------------------------ kda_forward without a workspace
@pytest.mark.parametrize("B,H,T,state", [(1, 2, 8197, True), (2, 3, 200, True), (3, 4, 130, False)])
def test_kda_forward_pooled_workspace_is_the_workspace_path(B, H, T, state):
    """kda_forward takes the same schedule on a workspace from the library's pool:
    bit-identical to kda_forward_ws with the fastest workspace."""
    w = I.scaled(I.PREFILL_B4_T16K_STATE if state else I.PREFILL_H16_T4K, B=B, H=H, T=T, seed=9900 + T)
    x = I.make_inputs(w, "cuda")
    out_w, s_w = _run(x, _ws(w))
    out_p, s_p = _run(x, None)
    assert torch.equal(out_p, out_w) and torch.equal(s_p, s_w)


# ------------------------------------------------------------ the pipelined schedule
def test_pipelined_schedule_every_workspace_size_bit_identical():
    """Few heads and at least 128 chunks: blocks of 64 chunks with the per-head chain
    beside the chunk-local kernel of the next block.  Batch > 1, a ragged tail and a
    carried state; the pipelined workspace, the smallest one that still pipelines
    (two blocks of 8 chunks), one below that (sequential blocks, same chain kernel)
    and the whole sequence's records all give the same bits, within the bar of the
    oracle."""
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=2, H=3, T=8192 + 61, seed=3131)     # 130 chunks
    x = I.make_inputs(w, "cuda")
    bh, rec = w.B * w.H, kda.workspace_bytes(1, 64, 1, 128, 128)
    state = bh * 128 * 128 * 4
    best = kda.workspace_bytes(w.B, w.T, w.H, 128, 128)
    assert best == 2 * 64 * bh * rec + state
    out_p, s_p = _run(x, _ws(w))
    _compare(x, out_p, s_p)
    for nbytes in (2 * 8 * bh * rec + state, 2 * 8 * bh * rec + state - 256, 130 * bh * rec):
        out_b, s_b = _run(x, _ws(w, nbytes))
        assert torch.equal(out_p, out_b) and torch.equal(s_p, s_b), nbytes


def test_pipelined_schedule_host_memory_path_bit_identical():
    """kda_forward_host on a pipelined shape picks the same chain kernel as the device
    call (the whole sequence's length decides), so the bits agree."""
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=1, H=2, T=8192 + 5, seed=3132)
    x = I.make_inputs(w, "cuda")
    out_d, s_d = _run(x, _ws(w))
    host = {n: x[n].cpu().pin_memory() for n in NAMES}
    out_h, s_h = kda.forward_host(*(host[n] for n in NAMES), x["initial_state"].cpu().pin_memory(),
                                  block_tokens=2048)
    kda.check_status()
    assert torch.equal(out_h, out_d.cpu()) and torch.equal(s_h, s_d.cpu())
