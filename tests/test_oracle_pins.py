"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

Each pin is chosen so that a plausible slip in the oracle (decay on the wrong
axis, prediction from the undecayed state, read before write, a wrong sign,
a dropped beta or scale, a transposed product) fails at least one of them.
Both oracle implementations (C and numpy) are pinned.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from tests.chunked_fp64 import chunked_forward

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
IMPLS = [pytest.param(oracle.forward, id="c"), pytest.param(oracle.forward_np, id="numpy")]


def _rand(seed, B=2, T=20, H=3, dk=8, dv=6, la_mu=-0.3, unit=True, s0=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk)).astype(np.float32)
    k = rng.standard_normal((B, T, H, dk)).astype(np.float32)
    if unit:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv)).astype(np.float32)
    la = (la_mu * rng.random((B, T, H, dk))).astype(np.float32)
    beta = rng.random((B, T, H)).astype(np.float32)
    S0 = rng.standard_normal((B, H, dk, dv)) if s0 else None
    return q, k, v, la, beta, S0


# ---------------------------------------------------------------- worked example
@pytest.mark.parametrize("fwd", IMPLS)
def test_worked_example_by_hand(fwd):
    """Hand-derived T=2, d=2 example (tests/golden/worked_example_d2_t2.json)."""
    g = json.load(open(os.path.join(GOLDEN, "worked_example_d2_t2.json")))
    shp = lambda a, d: np.array(a, dtype=np.float32).reshape(1, g["T"], 1, d)
    q, k, v = shp(g["q"], 2), shp(g["k"], 2), shp(g["v"], 2)
    la = np.log(shp(g["alpha"], 2).astype(np.float64)).astype(np.float32)
    beta = np.array(g["beta"], dtype=np.float32).reshape(1, g["T"], 1)
    S0 = np.array(g["initial_state"]).reshape(1, 1, 2, 2)
    out, sT = fwd(q, k, v, la, beta, S0, scale=g["scale"])
    # k2 = (0.6, 0.8) is not exact in fp32: allow its rounding (~1e-7 relative).
    np.testing.assert_allclose(out.reshape(2, 2), g["out"], rtol=0, atol=2e-6)
    np.testing.assert_allclose(sT.reshape(2, 2), g["final_state"], rtol=0, atol=2e-6)
    # default scale is 1/sqrt(dk) on the read
    out_d, _ = fwd(q, k, v, la, beta, S0)
    np.testing.assert_allclose(out_d, out / math.sqrt(2.0), rtol=1e-12, atol=0)


# ---------------------------------------------------------------- O1 pure decay
@pytest.mark.parametrize("fwd", IMPLS)
def test_beta_zero_is_pure_per_channel_decay(fwd):
    """beta = 0: nothing is written, S_t = Diag(prod alpha) S_0 row by row."""
    q, k, v, la, beta, S0 = _rand(1)
    beta[:] = 0
    out, sT = fwd(q, k, v, la, beta, S0)
    G = np.cumsum(la.astype(np.float64), axis=1)                       # [B,T,H,dk]
    S_t = np.exp(G)[..., :, None] * S0[:, None]                         # [B,T,H,dk,dv]
    o_ref = np.einsum("bthcx,bthc->bthx", S_t, q.astype(np.float64)) / math.sqrt(q.shape[-1])
    np.testing.assert_allclose(out, o_ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(sT, S_t[:, -1], rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- O2 linear attention
@pytest.mark.parametrize("fwd", IMPLS)
def test_small_beta_no_decay_is_linear_attention(fwd):
    """alpha = 1, S_0 = 0, beta = eps: o / eps -> scaled linear attention.

    The linear attention step S += v k^T, o = S q of the pages' first snippet,
    summed in closed form: o_t = scale * sum_{j<=t} (k_j . q_t) v_j.
    """
    q, k, v, la, beta, _ = _rand(2, T=24)
    la[:] = 0
    eps = 1e-7
    beta[:] = eps
    out, _ = fwd(q, k, v, la, beta, None)
    q64, k64, v64 = (x.astype(np.float64) for x in (q, k, v))
    T = q.shape[1]
    scores = np.einsum("bthc,bjhc->bhtj", q64, k64) * np.tril(np.ones((T, T)))
    lin = np.einsum("bhtj,bjhx->bthx", scores, v64) / math.sqrt(q.shape[-1])
    err = np.max(np.abs(out / eps - lin)) / np.max(np.abs(lin))
    assert err < 50 * eps * T


# ---------------------------------------------------------------- O3 DeltaNet
@pytest.mark.parametrize("fwd", IMPLS)
def test_no_decay_is_deltanet_in_value_by_key_layout(fwd):
    """alpha = 1: DeltaNet S' <- S'(I - beta k k^T) + beta v k^T with S' (dv x dk),
    read as scale * S' q (the projector form given on the technical deep dive)."""
    q, k, v, la, beta, S0 = _rand(3)
    la[:] = 0
    out, sT = fwd(q, k, v, la, beta, S0)
    B, T, H, dk = q.shape
    for b in range(B):
        for h in range(H):
            Sp = S0[b, h].T.copy()                                     # (dv, dk)
            for t in range(T):
                kt = k[b, t, h].astype(np.float64)
                bt = float(beta[b, t, h])
                Sp = Sp @ (np.eye(dk) - bt * np.outer(kt, kt)) + bt * np.outer(v[b, t, h].astype(np.float64), kt)
                np.testing.assert_allclose(out[b, t, h], Sp @ q[b, t, h].astype(np.float64) / math.sqrt(dk),
                                           rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(sT[b, h], Sp.T, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- O4 Gated DeltaNet
@pytest.mark.parametrize("fwd", IMPLS)
def test_scalar_decay_is_gated_deltanet(fwd):
    """All channels share alpha_t: S <- alpha_t (I - beta k k^T) S + beta k v^T."""
    q, k, v, la, beta, S0 = _rand(4)
    la[:] = la[..., :1]
    out, sT = fwd(q, k, v, la, beta, S0)
    B, T, H, dk = q.shape
    for b in range(B):
        for h in range(H):
            S = S0[b, h].copy()
            for t in range(T):
                kt = k[b, t, h].astype(np.float64)
                a = math.exp(float(la[b, t, h, 0]))
                bt = float(beta[b, t, h])
                S = a * (np.eye(dk) - bt * np.outer(kt, kt)) @ S + bt * np.outer(kt, v[b, t, h].astype(np.float64))
                np.testing.assert_allclose(out[b, t, h], S.T @ q[b, t, h].astype(np.float64) / math.sqrt(dk),
                                           rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(sT[b, h], S, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- O5 exact recall
@pytest.mark.parametrize("fwd", IMPLS)
def test_unit_write_recalls_value_exactly(fwd):
    """beta = 1 and |k| = 1: after each write S_t^T k_t = v_t for ANY alpha.

    Reading with q_t = k_t and scale = 1 gives o_t = S_t^T k_t = v_t, which also
    pins that the read happens after the write."""
    q, k, v, la, beta, S0 = _rand(5, la_mu=-2.0)
    k64 = k.astype(np.float64)
    k64 /= np.linalg.norm(k64, axis=-1, keepdims=True)
    kk = k64.astype(np.float32)
    beta[:] = 1.0
    out, _ = fwd(kk, kk, v, la, beta, S0, scale=1.0)
    # |kk| = 1 only to fp32 rounding, which bounds the deviation
    np.testing.assert_allclose(out, v.astype(np.float64), rtol=0, atol=5e-6)


# ---------------------------------------------------------------- O6 brute force
@pytest.mark.parametrize("fwd", IMPLS)
def test_unrolled_matrix_products_tiny(fwd):
    """T <= 8: S_t = M_t ... M_1 S_0 + sum_j M_t ... M_{j+1} beta_j k_j v_j^T,
    M_t = (I - beta_t k_t k_t^T) Diag(alpha_t), and o_t = scale S_t^T q_t."""
    q, k, v, la, beta, S0 = _rand(6, B=1, T=8, H=2, dk=5, dv=4, la_mu=-1.0, unit=False)
    out, sT = fwd(q, k, v, la, beta, S0)
    T, dk = q.shape[1], q.shape[-1]
    for h in range(2):
        Ms = []
        for t in range(T):
            kt = k[0, t, h].astype(np.float64)
            Ms.append((np.eye(dk) - float(beta[0, t, h]) * np.outer(kt, kt)) @ np.diag(np.exp(la[0, t, h].astype(np.float64))))
        for t in range(T):
            P = np.eye(dk)
            for s in range(t, -1, -1):
                P = P @ Ms[s]
            S_t = P @ S0[0, h]
            for j in range(t + 1):
                Pj = np.eye(dk)
                for s in range(t, j, -1):
                    Pj = Pj @ Ms[s]
                S_t = S_t + Pj @ (float(beta[0, j, h]) * np.outer(k[0, j, h].astype(np.float64),
                                                               v[0, j, h].astype(np.float64)))
            np.testing.assert_allclose(out[0, t, h], S_t.T @ q[0, t, h].astype(np.float64) / math.sqrt(dk),
                                       rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(sT[0, h], S_t, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- O7 chunk algebra
@pytest.mark.parametrize("C,T", [(64, 200), (32, 96), (16, 37), (8, 1)])
def test_chunked_form_equals_recurrence(C, T):
    """The WY/UT chunk algebra the CUDA prefill uses equals the recurrence."""
    q, k, v, la, beta, S0 = _rand(7, B=1, T=T, H=2, dk=16, dv=12, la_mu=-0.2)
    o_ref, s_ref = oracle.forward(q, k, v, la, beta, S0)
    o_ch, s_ch = chunked_forward(q, k, v, la, beta, S0, C=C)
    assert oracle.parity_error(o_ch, o_ref) < 1e-12
    assert oracle.parity_error(s_ch, s_ref) < 1e-12


# ---------------------------------------------------------------- O8 state carry
@pytest.mark.parametrize("fwd", IMPLS)
def test_split_linearity_and_column_independence(fwd):
    q, k, v, la, beta, S0 = _rand(8, T=30)
    o, s = fwd(q, k, v, la, beta, S0)
    # split invariance: run 0..11, carry the state, run 12..29
    o1, s1 = fwd(q[:, :12], k[:, :12], v[:, :12], la[:, :12], beta[:, :12], S0)
    o2, s2 = fwd(q[:, 12:], k[:, 12:], v[:, 12:], la[:, 12:], beta[:, 12:], s1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s2, s, rtol=1e-12, atol=1e-13)
    # outputs and state are linear in (V, S_0) jointly for fixed q, k, alpha, beta
    # dyadic values keep 2 v - 3 v2 exact in fp32, the oracle's input type
    rng = np.random.default_rng(9)
    v = (np.round(v * 1024) / 1024).astype(np.float32)
    o, s = fwd(q, k, v, la, beta, S0)
    v2 = (np.round(rng.standard_normal(v.shape) * 1024) / 1024).astype(np.float32)
    S02 = rng.standard_normal(S0.shape)
    ob, sb = fwd(q, k, v2, la, beta, S02)
    oc, sc = fwd(q, k, (2 * v - 3 * v2).astype(np.float32), la, beta, 2 * S0 - 3 * S02)
    np.testing.assert_allclose(oc, 2 * o - 3 * ob, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(sc, 2 * s - 3 * sb, rtol=1e-10, atol=1e-11)
    # value columns evolve independently: column x of S and o sees only column x of v, S_0
    od, sd = fwd(q, k, v[..., 2:3].copy(), la, beta, S0[..., 2:3].copy())
    np.testing.assert_allclose(od[..., 0], o[..., 2], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(sd[..., 0], s[..., 2], rtol=1e-12, atol=1e-13)


def test_c_and_numpy_oracles_agree():
    q, k, v, la, beta, S0 = _rand(10, B=2, T=40, H=3, dk=16, dv=16)
    oa, sa = oracle.forward(q, k, v, la, beta, S0, nthreads=3)
    ob, sb = oracle.forward_np(q, k, v, la, beta, S0)
    np.testing.assert_allclose(oa, ob, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(sa, sb, rtol=1e-12, atol=1e-13)


def test_empty_sequence_returns_initial_state():
    q, k, v, la, beta, S0 = _rand(11, T=0)
    for fwd in (oracle.forward, oracle.forward_np):
        o, s = fwd(q, k, v, la, beta, S0)
        assert o.shape == (2, 0, 3, 6)
        np.testing.assert_array_equal(s, S0)
        o, s = fwd(q, k, v, la, beta, None)
        np.testing.assert_array_equal(s, np.zeros_like(S0))


def test_parity_metric():
    ref = np.array([1.0, -1.0, 1.0, -1.0])
    assert oracle.parity_error(ref + np.array([0, 0, 0.002, 0]), ref) == pytest.approx(0.002)
    assert oracle.parity_error(np.zeros(0), np.zeros(0)) == 0.0


# ---------------------------------------------------------------- O9 scalar-gate entry
def test_gdn_forward_is_the_gated_deltanet_recurrence():
    """oracle.gdn_forward with a [B,T,H] gate against the textbook Gated DeltaNet
    step S <- alpha_t (I - beta k k^T) S + beta k v^T, read S^T q / sqrt(dk); with
    no gate, against the DeltaNet step (alpha = 1)."""
    q, k, v, la, beta, S0 = _rand(21, T=17, dk=8, dv=5)
    g = np.ascontiguousarray(la[..., 0] - 0.5)            # [B,T,H], distinct per token and head
    B, T, H, dk = q.shape
    for gate in (g, None):
        out, sT = oracle.gdn_forward(q, k, v, gate, beta, S0)
        for b in range(B):
            for h in range(H):
                S = S0[b, h].copy()
                for t in range(T):
                    kt = k[b, t, h].astype(np.float64)
                    a = 1.0 if gate is None else math.exp(float(gate[b, t, h]))
                    bt = float(beta[b, t, h])
                    S = a * (np.eye(dk) - bt * np.outer(kt, kt)) @ S + bt * np.outer(kt, v[b, t, h].astype(np.float64))
                    np.testing.assert_allclose(out[b, t, h], S.T @ q[b, t, h].astype(np.float64) / math.sqrt(dk),
                                               rtol=1e-11, atol=1e-12)
                np.testing.assert_allclose(sT[b, h], S, rtol=1e-11, atol=1e-12)


def test_gdn_forward_rotation_invariance():
    """A decay shared by all key channels commutes with any rotation U of key
    space: (U q, U k, U S0) gives the same outputs and U S_T.  A per-channel
    decay does not, so this fails if the scalar gate reaches the channels
    unevenly."""
    q, k, v, la, beta, S0 = _rand(22, T=24, dk=8, dv=4)
    g = np.ascontiguousarray(-0.2 - la[..., 0])
    U, _ = np.linalg.qr(np.random.default_rng(7).standard_normal((8, 8)))
    rot = lambda x: np.einsum("ij,bthj->bthi", U, x.astype(np.float64)).astype(np.float32)
    out, sT = oracle.gdn_forward(q, k, v, g, beta, S0)
    out_r, sT_r = oracle.gdn_forward(rot(q), rot(k), v, g, beta, np.einsum("ij,bhjx->bhix", U, S0))
    # the rotated q, k are rounded to fp32: agreement to fp32 input precision
    assert oracle.parity_error(out_r, out) < 2e-5
    assert oracle.parity_error(sT_r, np.einsum("ij,bhjx->bhix", U, sT)) < 2e-5
    # the same property fails for KDA's per-channel gate
    out_c, _ = oracle.forward(q, k, v, la * 8, beta, S0)
    out_cr, _ = oracle.forward(rot(q), rot(k), v, la * 8, beta, np.einsum("ij,bhjx->bhix", U, S0))
    assert oracle.parity_error(out_cr, out_c) > 1e-2


def test_gdn_forward_empty_and_shape_check():
    q, k, v, la, beta, S0 = _rand(23, T=0)
    o, s = oracle.gdn_forward(q, k, v, la[..., 0], beta, S0)
    assert o.shape == (2, 0, 3, 6)
    np.testing.assert_array_equal(s, S0)
    with pytest.raises(ValueError):
        oracle.gdn_forward(q, k, v, la, beta, S0)          # a per-channel gate is not accepted


# ---------------------------------------------------------------- O10 raw activations
def _raw(seed, B=2, T=19, H=3, dk=8, dv=5):
    rng = np.random.default_rng(seed)
    q = (3.0 * rng.standard_normal((B, T, H, dk))).astype(np.float32)
    k = (0.5 * rng.standard_normal((B, T, H, dk))).astype(np.float32)
    v = rng.standard_normal((B, T, H, dv)).astype(np.float32)
    x = (2.0 + rng.standard_normal((B, T, H, dk))).astype(np.float32)
    beta = rng.random((B, T, H)).astype(np.float32)
    S0 = rng.standard_normal((B, H, dk, dv))
    return q, k, v, x, beta, S0


def test_raw_gate_is_log_of_sigmoid():
    """gate pre-activations x give the same result as log alpha = log(1 / (1 + e^-x))
    written out directly (unit q, k, so normalisation is the identity)."""
    q, k, v, x, beta, S0 = _raw(31)
    q = (q / np.linalg.norm(q.astype(np.float64), axis=-1, keepdims=True)).astype(np.float32)
    k = (k / np.linalg.norm(k.astype(np.float64), axis=-1, keepdims=True)).astype(np.float32)
    la = np.log(1.0 / (1.0 + np.exp(-x.astype(np.float64))))
    o_ref, s_ref = oracle.forward(q, k, v, la, beta, S0)
    o, s = oracle.forward_raw(q, k, v, x, beta, S0, logsigmoid_gate=True, normalize_qk=False)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=2e-6 * np.abs(o_ref).max())
    np.testing.assert_allclose(s, s_ref, rtol=0, atol=2e-6 * np.abs(s_ref).max())


def test_raw_normalisation_is_per_row_and_scale_free():
    """Rescaling each (b, t, h) row of q and k by a positive factor changes nothing;
    unit rows reproduce forward(); the result depends on q, k only through q/|q|, k/|k|."""
    q, k, v, x, beta, S0 = _raw(32)
    la = -np.logaddexp(0.0, -x.astype(np.float64))
    rng = np.random.default_rng(5)
    cq = rng.uniform(0.1, 10.0, q.shape[:-1] + (1,)).astype(np.float32)
    ck = rng.uniform(0.1, 10.0, k.shape[:-1] + (1,)).astype(np.float32)
    o1, s1 = oracle.forward_raw(q, k, v, la, beta, S0, logsigmoid_gate=False, normalize_qk=True)
    o2, s2 = oracle.forward_raw(q * cq, k * ck, v, la, beta, S0, logsigmoid_gate=False, normalize_qk=True)
    assert oracle.parity_error(o2, o1) < 1e-5 and oracle.parity_error(s2, s1) < 1e-5
    qn = q / np.linalg.norm(q.astype(np.float64), axis=-1, keepdims=True)
    kn = k / np.linalg.norm(k.astype(np.float64), axis=-1, keepdims=True)
    o3, s3 = oracle.forward(qn, kn, v, la, beta, S0)
    assert oracle.parity_error(o3, o1) < 1e-5 and oracle.parity_error(s3, s1) < 1e-5
    # and the factors matter without normalisation
    o4, _ = oracle.forward_raw(q * cq, k * ck, v, la, beta, S0, logsigmoid_gate=False, normalize_qk=False)
    assert oracle.parity_error(o4, o1) > 1e-2


def test_raw_zero_key_row_writes_nothing():
    q, k, v, x, beta, S0 = _raw(33, B=1, H=1, T=6)
    k[0, 3, 0] = 0.0
    o, s = oracle.forward_raw(q, k, v, x, beta, S0)
    assert np.isfinite(o).all() and np.isfinite(s).all()
    # token 3 with a zero key only decays the state: same as beta = 0 there
    b2 = beta.copy()
    b2[0, 3, 0] = 0.0
    k2 = k.copy()
    k2[0, 3, 0] = 1.0
    o2, s2 = oracle.forward_raw(q, k2, v, x, b2, S0)
    np.testing.assert_allclose(s, s2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(o[0, 4:], o2[0, 4:], rtol=1e-12, atol=1e-12)
