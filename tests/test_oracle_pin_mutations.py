"""The oracle pins catch plausible mistakes.

Each case below is the numpy oracle with one deliberate slip planted in a local
copy (on the CPU; the real oracle is untouched).  Every slip must make at least
one pin in test_oracle_pins fail.
"""
import math

import numpy as np
import pytest

import oracle
from tests import test_oracle_pins as pins


def _make(mutation):
    def fwd(q, k, v, log_alpha, beta, initial_state=None, scale=None):
        qf, kf, vf, af, bf = (oracle._as_f32(x).astype(np.float64) for x in (q, k, v, log_alpha, beta))
        B, T, H, dk = qf.shape
        dv = vf.shape[-1]
        if scale is None:
            scale = 1.0 / math.sqrt(dk)
        if mutation == "no_scale":
            scale = 1.0
        S = np.zeros((B, H, dk, dv)) if initial_state is None else oracle._as_f64(initial_state).copy()
        out = np.empty((B, T, H, dv))
        for t in range(T):
            alpha = af[:, t] if mutation == "alpha_not_exp" else np.exp(af[:, t])
            if mutation == "read_before_write":
                pre = np.einsum("bhcx,bhc->bhx", S * alpha[..., :, None], qf[:, t])
            S_old = S
            if mutation == "decay_value_axis":
                S = S * alpha[..., None, :dv] if dv <= dk else S
            else:
                S = S * alpha[..., :, None]
            src = S_old if mutation == "predict_undecayed" else S
            p = np.einsum("bhcx,bhc->bhx", src, kf[:, t])
            e = vf[:, t] - p if mutation == "no_beta" else bf[:, t, :, None] * (vf[:, t] - p)
            if mutation == "error_sign":
                e = -e
            S = S + kf[:, t][..., :, None] * e[..., None, :]
            if mutation == "transposed_read" and dk == dv:
                o = np.einsum("bhxc,bhc->bhx", S, qf[:, t])
            elif mutation == "read_before_write":
                o = pre
            else:
                o = np.einsum("bhcx,bhc->bhx", S, qf[:, t])
            out[:, t] = scale * o
        return out, S
    return fwd


PIN_TESTS = [pins.test_worked_example_by_hand, pins.test_beta_zero_is_pure_per_channel_decay,
             pins.test_small_beta_no_decay_is_linear_attention,
             pins.test_no_decay_is_deltanet_in_value_by_key_layout,
             pins.test_scalar_decay_is_gated_deltanet, pins.test_unit_write_recalls_value_exactly,
             pins.test_unrolled_matrix_products_tiny]


@pytest.mark.parametrize("mutation", ["decay_value_axis", "predict_undecayed", "read_before_write",
                                      "error_sign", "no_beta", "no_scale", "transposed_read",
                                      "alpha_not_exp"])
def test_some_pin_fails_on_planted_mistake(mutation):
    fwd = _make(mutation)
    failed = []
    for t in PIN_TESTS:
        try:
            t(fwd)
        except AssertionError:
            failed.append(t.__name__)
    assert failed, "no pin caught the planted mistake %r" % mutation


def test_unmutated_copy_passes_every_pin():
    fwd = _make("none")
    for t in PIN_TESTS:
        t(fwd)


def _make_gdn(mutation):
    """oracle.gdn_forward with one slip in how the [B,T,H] gate reaches the channels."""
    def gdn(q, k, v, log_alpha, beta, initial_state=None, scale=None, nthreads=0):
        qf = oracle._as_f32(q)
        B, T, H, dk = qf.shape
        g = np.zeros((B, T, H), np.float32) if log_alpha is None else oracle._as_f32(log_alpha)
        if mutation == "first_channel_only":
            la = np.zeros((B, T, H, dk), np.float32)
            la[..., 0] = g
        elif mutation == "token_head_swapped":
            la = np.repeat(g.reshape(B, H, T).transpose(0, 2, 1)[..., None], dk, axis=-1)
        elif mutation == "gate_not_applied":
            la = np.zeros((B, T, H, dk), np.float32)
        else:
            la = np.repeat(g[..., None], dk, axis=-1)
        return oracle.forward(qf, k, v, np.ascontiguousarray(la), beta, initial_state, scale=scale)
    return gdn


GDN_PINS = [pins.test_gdn_forward_is_the_gated_deltanet_recurrence, pins.test_gdn_forward_rotation_invariance]


@pytest.mark.parametrize("mutation", ["first_channel_only", "token_head_swapped", "gate_not_applied"])
def test_some_gdn_pin_fails_on_planted_mistake(mutation, monkeypatch):
    monkeypatch.setattr(oracle, "gdn_forward", _make_gdn(mutation))
    failed = 0
    for pin in GDN_PINS:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed > 0, "no scalar-gate pin caught %s" % mutation


def test_unmutated_gdn_copy_passes_every_pin(monkeypatch):
    monkeypatch.setattr(oracle, "gdn_forward", _make_gdn("none"))
    for pin in GDN_PINS:
        pin()


def _make_raw(mutation):
    """oracle.forward_raw with one slip in the steps before the path."""
    def raw(q, k, v, gate, beta, initial_state=None, logsigmoid_gate=True, normalize_qk=True, scale=None,
            nthreads=0):
        q64, k64, g64 = (oracle._as_f64(x) for x in (q, k, gate))
        if normalize_qk:
            axis = 1 if mutation == "norm_over_tokens" else -1
            q64 = q64 / np.linalg.norm(q64, axis=axis, keepdims=True)
            k64 = k64 / np.linalg.norm(k64, axis=axis, keepdims=True)
        if logsigmoid_gate:
            la = np.log(1.0 / (1.0 + np.exp(-g64))) if mutation != "sigmoid_not_logged" else 1.0 / (1.0 + np.exp(-g64)) - 1.0
        else:
            la = g64
        return oracle.forward(q64, k64, v, la, beta, initial_state, scale=scale)
    return raw


RAW_PINS = [pins.test_raw_gate_is_log_of_sigmoid, pins.test_raw_normalisation_is_per_row_and_scale_free]


@pytest.mark.parametrize("mutation", ["norm_over_tokens", "sigmoid_not_logged"])
def test_some_raw_pin_fails_on_planted_mistake(mutation, monkeypatch):
    monkeypatch.setattr(oracle, "forward_raw", _make_raw(mutation))
    failed = 0
    for pin in RAW_PINS:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed > 0, "no raw-activation pin caught %s" % mutation


def test_unmutated_raw_copy_passes_every_pin(monkeypatch):
    monkeypatch.setattr(oracle, "forward_raw", _make_raw("none"))
    for pin in RAW_PINS:
        pin()


def _make_bwd(mutation):
    """oracle.backward with one slip planted in the differentiated recurrence."""
    def bwd(q, k, v, log_alpha, beta, d_out, initial_state=None, d_final_state=None, scale=None, segment=64):
        import torch
        ex = lambda x: torch.from_numpy(oracle._as_f32(x).astype(np.float64))
        qt, kt, vt, at, bt = (ex(x).requires_grad_(True) for x in (q, k, v, log_alpha, beta))
        B, T, H, dk = qt.shape
        dv = vt.shape[-1]
        sc = 1.0 if mutation == "no_scale" else (1.0 / math.sqrt(dk) if scale is None else scale)
        s0 = (torch.zeros((B, H, dk, dv), dtype=torch.float64) if initial_state is None
              else torch.from_numpy(oracle._as_f64(initial_state)).clone()).requires_grad_(True)
        d_o = torch.from_numpy(oracle._as_f64(d_out))
        d_s = (torch.zeros((B, H, dk, dv), dtype=torch.float64)
               if d_final_state is None or mutation == "final_cotangent_dropped"
               else torch.from_numpy(oracle._as_f64(d_final_state)))
        S, loss = s0, torch.zeros((), dtype=torch.float64)
        for t0 in range(0, T, segment):
            if mutation == "segments_restart":
                S = s0
            for t in range(t0, min(T, t0 + segment)):
                Sd = S * torch.exp(at[:, t]).unsqueeze(-1)
                p = torch.einsum("bhcx,bhc->bhx", S if mutation == "predict_undecayed" else Sd, kt[:, t])
                e = bt[:, t].unsqueeze(-1) * (vt[:, t] - p)
                Sn = Sd + kt[:, t].unsqueeze(-1) * e.unsqueeze(-2)
                o = sc * torch.einsum("bhcx,bhc->bhx", Sd if mutation == "read_before_write" else Sn, qt[:, t])
                loss = loss + (o * d_o[:, t]).sum()
                S = Sn
        loss = loss + (S * d_s).sum()
        g = torch.autograd.grad(loss, [qt, kt, vt, at, bt, s0], allow_unused=True)
        names = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dinitial_state")
        ref = (qt, kt, vt, at, bt, s0)
        return {n: (gi if gi is not None else torch.zeros_like(r)).detach().numpy()
                for n, gi, r in zip(names, g, ref)}
    return bwd


from tests import test_oracle_backward_pins as bpins  # noqa: E402

BWD_PINS = [bpins.test_backward_matches_finite_differences, bpins.test_backward_beta_zero_closed_form]


@pytest.mark.parametrize("mutation", ["final_cotangent_dropped", "predict_undecayed", "segments_restart",
                                      "read_before_write", "no_scale"])
def test_some_backward_pin_fails_on_planted_mistake(mutation, monkeypatch):
    monkeypatch.setattr(oracle, "backward", _make_bwd(mutation))
    failed = 0
    for pin in BWD_PINS:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed > 0, "no backward pin caught %s" % mutation


def test_unmutated_backward_copy_passes_every_pin(monkeypatch):
    monkeypatch.setattr(oracle, "backward", _make_bwd("none"))
    for pin in BWD_PINS:
        pin()
