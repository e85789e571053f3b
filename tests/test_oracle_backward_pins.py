"""Pins of the oracle's backward (the gradients of the KDA forward).

oracle.backward differentiates the token recurrence with torch.autograd.  It is
pinned here to things outside itself:

* B1  central finite differences of the numpy forward (oracle.forward_np, pinned
      by test_oracle_pins) along random directions, for every input;
* B2  the closed form of the gradients when beta = 0 (pure per-channel decay:
      S_t = Diag(Gamma_t) S_0, no write), written directly, without a recurrence;
* B3  the empty sequence: only the initial state has a gradient, the final-state
      cotangent itself.

A planted mistake in a copy of the backward fails one of them
(test_oracle_pin_mutations).

The last test runs the other way: the pinned oracle checks the chunkwise gradient
algebra (tests/chunked_fp64.py) that a chunked backward follows.
"""
import math

import numpy as np
import pytest

import oracle
from tests.chunked_fp64 import chunked_backward

NAMES = ("q", "k", "v", "log_alpha", "beta", "initial_state")
GRAD = {"q": "dq", "k": "dk", "v": "dv", "log_alpha": "dlog_alpha", "beta": "dbeta",
        "initial_state": "dinitial_state"}


def _draw(seed, B=1, T=13, H=2, dk=6, dv=5, beta_zero=False):
    rng = np.random.default_rng(seed)
    f32 = lambda a: np.asarray(a, dtype=np.float32)
    x = {
        "q": f32(rng.standard_normal((B, T, H, dk)) / math.sqrt(dk)),
        "k": f32(rng.standard_normal((B, T, H, dk)) / math.sqrt(dk)),
        "v": f32(rng.standard_normal((B, T, H, dv))),
        "log_alpha": f32(-np.abs(rng.normal(0.2, 0.2, (B, T, H, dk)))),
        "beta": f32(np.zeros((B, T, H)) if beta_zero else rng.uniform(0.1, 0.9, (B, T, H))),
        "initial_state": f32(0.5 * rng.standard_normal((B, H, dk, dv))),
    }
    d_out = rng.standard_normal((B, T, H, dv))
    d_fin = rng.standard_normal((B, H, dk, dv))
    return x, d_out, d_fin


def _loss(x, d_out, d_fin):
    o, s = oracle.forward_np(*(x[n] for n in NAMES), exact64=True)
    return float((o * d_out).sum() + (s * d_fin).sum())


def test_backward_matches_finite_differences():
    """B1: <grad, u> equals (L(x + h u) - L(x - h u)) / 2h for every input."""
    x, d_out, d_fin = _draw(1)
    # segments of 5 tokens: the state carried between checkpointed segments is pinned too
    g = oracle.backward(*(x[n] for n in NAMES[:5]), d_out, x["initial_state"], d_fin, segment=5)
    rng = np.random.default_rng(2)
    h = 1e-5
    for n in NAMES:
        u = rng.standard_normal(x[n].shape)
        xp = {m: x[m].astype(np.float64) for m in NAMES}
        xm = {m: x[m].astype(np.float64) for m in NAMES}
        xp[n] = xp[n] + h * u
        xm[n] = xm[n] - h * u
        fd = (_loss(xp, d_out, d_fin) - _loss(xm, d_out, d_fin)) / (2 * h)
        an = float((g[GRAD[n]] * u).sum())
        assert abs(fd - an) <= 1e-6 * (1.0 + abs(an)), (n, fd, an)


def test_backward_beta_zero_closed_form():
    """B2: with beta = 0 the state is Diag(Gamma_t) S_0 (Gamma_t = exp of the running
    sum of log alpha) and every gradient has a direct formula."""
    x, d_out, d_fin = _draw(3, B=2, T=17, H=2, dk=7, dv=5, beta_zero=True)
    g = oracle.backward(*(x[n] for n in NAMES[:5]), d_out, x["initial_state"], d_fin, segment=4)
    q, k, v, la = (x[n].astype(np.float64) for n in ("q", "k", "v", "log_alpha"))
    S0 = x["initial_state"].astype(np.float64)
    B, T, H, dk = q.shape
    sc = 1.0 / math.sqrt(dk)
    Gam = np.exp(np.cumsum(la, axis=1))                                   # [B,T,H,dk]
    S0dO = np.einsum("bhcx,bthx->bthc", S0, d_out)                        # (S_0 dO_t)_c
    # dq_t = scale Diag(Gamma_t) S_0 dO_t; dk = dv = 0
    assert np.allclose(g["dq"], sc * Gam * S0dO, rtol=1e-12, atol=1e-12)
    assert np.abs(g["dk"]).max() < 1e-12 and np.abs(g["dv"]).max() < 1e-12
    # dS_0 = sum_t scale Diag(Gamma_t) q_t dO_t^T + Diag(Gamma_last) dS_T
    dS0 = sc * np.einsum("bthc,bthx->bhcx", Gam * q, d_out) + Gam[:, -1][..., None] * d_fin
    assert np.allclose(g["dinitial_state"], dS0, rtol=1e-12, atol=1e-12)
    # d log alpha_t = sum over tau >= t of dL/dG_tau
    dG = sc * q * Gam * S0dO
    dG[:, -1] += Gam[:, -1] * np.einsum("bhcx,bhcx->bhc", S0, d_fin)
    dla = np.flip(np.cumsum(np.flip(dG, axis=1), axis=1), axis=1)
    assert np.allclose(g["dlog_alpha"], dla, rtol=1e-10, atol=1e-12)
    # dbeta_t = k_t^T (dL/dS_t) (v_t - p_t), dL/dS_t = sum_{tau >= t} Diag(Gamma_tau / Gamma_t)
    # scale q_tau dO_tau^T + Diag(Gamma_last / Gamma_t) dS_T, p_t = (Diag(Gamma_t) S_0)^T k_t
    dbeta = np.zeros((B, T, H))
    for b in range(B):
        for hh in range(H):
            for t in range(T):
                adj = (Gam[b, -1, hh] / Gam[b, t, hh])[:, None] * d_fin[b, hh]
                for tau in range(t, T):
                    adj = adj + sc * np.outer(Gam[b, tau, hh] / Gam[b, t, hh] * q[b, tau, hh], d_out[b, tau, hh])
                p = (Gam[b, t, hh][:, None] * S0[b, hh]).T @ k[b, t, hh]
                dbeta[b, t, hh] = k[b, t, hh] @ adj @ (v[b, t, hh] - p)
    assert np.allclose(g["dbeta"], dbeta, rtol=1e-10, atol=1e-12)


def test_backward_empty_sequence():
    """B3: T = 0 leaves only the initial state, whose gradient is the cotangent."""
    x, d_out, d_fin = _draw(4, T=0)
    g = oracle.backward(*(x[n] for n in NAMES[:5]), d_out, x["initial_state"], d_fin)
    assert np.array_equal(g["dinitial_state"], d_fin)
    assert g["dq"].shape == x["q"].shape and g["dbeta"].shape == x["beta"].shape


def test_backward_segment_length_does_not_change_the_gradient():
    x, d_out, d_fin = _draw(5, T=21)
    ref = oracle.backward(*(x[n] for n in NAMES[:5]), d_out, x["initial_state"], d_fin, segment=64)
    for seg in (1, 4):
        g = oracle.backward(*(x[n] for n in NAMES[:5]), d_out, x["initial_state"], d_fin, segment=seg)
        for n in GRAD.values():
            assert np.allclose(g[n], ref[n], rtol=1e-12, atol=1e-14), (seg, n)


def test_backward_without_state_arguments():
    x, d_out, _ = _draw(6, T=9)
    g = oracle.backward(*(x[n] for n in NAMES[:5]), d_out)
    assert g["dinitial_state"].shape == x["initial_state"].shape
    g0 = oracle.backward(*(x[n] for n in NAMES[:5]), np.zeros_like(d_out))
    assert all(np.abs(g0[n]).max() == 0.0 for n in GRAD.values())


@pytest.mark.parametrize("C,T,states", [(64, 150, True), (16, 37, True), (8, 21, False), (5, 13, True),
                                        (1, 6, False)])
def test_chunked_gradient_algebra_equals_the_oracle(C, T, states):
    """The chunkwise gradient (tests/chunked_fp64.py: a serial dS chain that is the
    forward chain transposed, everything else chunk-parallel through the WY
    factors) equals the pinned gradients of the token recurrence in fp64, over
    whole chunks and a ragged last chunk."""
    x, d_out, d_fin = _draw(11 + C, T=T, H=2, dk=8, dv=6)
    s0, dfin = (x["initial_state"], d_fin) if states else (None, None)
    ref = oracle.backward(*(x[n] for n in NAMES[:5]), d_out, s0, dfin)
    got = chunked_backward(*(x[n] for n in NAMES[:5]), d_out, s0, dfin, C=C)
    for n in GRAD.values():
        assert oracle.parity_error(got[n], ref[n]) < 1e-12, n
