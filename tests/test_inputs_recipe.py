"""The seeded input generators follow the stated recipe: reproducible draws, unit
q and k rows, a sigmoid retention gate given as its log, a sigmoid write
strength, the stated distributions of the pre-activations and of the carried
state, and the library's layouts.  Sizes are cut down along T (or the decode
steps) so that the checks run in seconds on the host."""
import math

import pytest
import torch

from gated_delta_rule_109_b200 import inputs as I


def small(w):
    return I.scaled(w, steps=8) if w.is_decode else I.scaled(w, T=min(w.T, 512))


@pytest.mark.parametrize("w", I.WORKLOADS, ids=lambda w: w.name)
def test_shapes_dtypes_and_reproducibility(w):
    w = small(w)
    a, b = I.make_inputs(w), I.make_inputs(w)
    lead = (w.steps, w.B, w.H) if w.is_decode else (w.B, w.T, w.H)
    assert a["q"].shape == lead + (w.dk,) and a["k"].shape == lead + (w.dk,)
    assert a["v"].shape == lead + (w.dv,)
    assert a["log_alpha"].shape == lead + (w.dk,) and a["beta"].shape == lead
    assert a["q"].dtype == a["k"].dtype == a["v"].dtype == w.torch_dtype
    assert a["log_alpha"].dtype == a["beta"].dtype == torch.float32
    if w.state_sd is None:
        assert a["initial_state"] is None
    else:
        assert a["initial_state"].shape == (w.B, w.H, w.dk, w.dv)
        assert a["initial_state"].dtype == torch.float32
    for key in a:
        if a[key] is not None:
            assert a[key].is_contiguous()
            assert torch.equal(a[key], b[key]), key
    c = I.make_inputs(I.scaled(w, seed=w.seed + 100))
    assert not torch.equal(a["q"], c["q"])


@pytest.mark.parametrize("w", I.WORKLOADS, ids=lambda w: w.name)
def test_query_and_key_rows_are_unit_length(w):
    x = I.make_inputs(small(w))
    # normalised in fp32, then rounded once to the input dtype
    tol = 1e-6 if w.dtype == "f32" else 2 ** -8 * 2
    for name in ("q", "k"):
        n = x[name].float().norm(dim=-1)
        assert (n - 1).abs().max().item() < tol, name


@pytest.mark.parametrize("w", I.WORKLOADS, ids=lambda w: w.name)
def test_gate_and_write_strength_distributions(w):
    w = small(w)
    x = I.make_inputs(w)
    la = x["log_alpha"].double()
    assert (la < 0).all() and torch.isfinite(la).all()
    # invert the log-sigmoid: x_alpha = la - log(1 - e^la)
    xa = la - torch.log(-torch.expm1(la))
    n = xa.numel()
    assert abs(xa.mean().item() - w.alpha_mu) < 6 * w.alpha_sd / math.sqrt(n) + 1e-3
    assert abs(xa.std().item() / w.alpha_sd - 1) < 0.05
    bt = x["beta"].double()
    assert ((bt > 0) & (bt < 1)).all()
    xb = torch.log(bt / (1 - bt))
    nb = xb.numel()
    assert abs(xb.mean().item() - w.beta_mu) < 6 * w.beta_sd / math.sqrt(nb) + 1e-3
    assert abs(xb.std().item() / w.beta_sd - 1) < 0.1
    v = x["v"].double()
    assert abs(v.mean().item()) < 6 / math.sqrt(v.numel()) + 1e-3
    assert abs(v.std().item() - 1) < 0.05
    if w.state_sd is not None:
        s = x["initial_state"].double()
        assert abs(s.std().item() / w.state_sd - 1) < 0.02
        assert abs(s.mean().item()) < 6 * w.state_sd / math.sqrt(s.numel())


@pytest.mark.parametrize("w", [wl for wl in I.WORKLOADS if not wl.is_decode], ids=lambda w: w.name)
def test_raw_inputs_are_the_same_draws_before_activation_and_normalisation(w):
    w = small(w)
    x, r = I.make_inputs(w), I.make_raw_inputs(w)
    assert torch.equal(x["v"], r["v"]) and torch.equal(x["beta"], r["beta"])
    if w.state_sd is not None:
        assert torch.equal(x["initial_state"], r["initial_state"])
    # the gate pre-activations give log_alpha through the fp64 log-sigmoid
    la = torch.nn.functional.logsigmoid(r["gate"].double()).float()
    assert torch.equal(la, x["log_alpha"])
    if w.dtype == "f32":
        # raw rows are the unnormalised draws: normalising them gives q and k back
        for name in ("q", "k"):
            raw = r[name]
            assert torch.allclose(raw / raw.norm(dim=-1, keepdim=True), x[name], atol=1e-6)
    else:
        # bf16 raw rows point the same way as the normalised ones
        for name in ("q", "k"):
            cos = torch.nn.functional.cosine_similarity(r[name].float(), x[name].float(), dim=-1)
            assert cos.min().item() > 0.999


def test_decode_steps_override():
    w = I.scaled(I.DECODE_B256, B=2, H=2)
    x = I.make_inputs(w, steps=3)
    assert x["q"].shape == (3, 2, 2, w.dk)
    with pytest.raises(ValueError):
        I.make_raw_inputs(w)
