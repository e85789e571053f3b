"""Time-axis split on one device: a sequence cut into R segments, each run from a
zero state (kda_segment_local), their start states composed
(kda_segment_start_state) and their outputs corrected (kda_segment_correct),
equals the prefill of the whole sequence.  No kernel waits on another; the
segments run one after another."""
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


def _split_run(x, cuts):
    B, T, H, dk = x["q"].shape
    bounds = [0] + list(cuts) + [T]
    outs, Ps, Fs, wss, segs = [], [], [], [], []
    for r in range(len(bounds) - 1):
        a, b = bounds[r], bounds[r + 1]
        seg = {n: x[n][:, a:b].contiguous() for n in NAMES}
        ws = kda.make_workspace(B, b - a, H, 128, 128, segment=True)
        o, lf, P = kda.segment_local(*(seg[n] for n in NAMES), x["initial_state"] if r == 0 else None, workspace=ws)
        outs.append(o); Ps.append(P); Fs.append(lf); wss.append(ws)
    final = Fs[0]
    for r in range(1, len(outs)):
        start = kda.segment_start_state(torch.stack(Ps[:r]), torch.stack(Fs[:r]))
        final = kda.segment_correct(start, Fs[r], outs[r], workspace=wss[r])
    torch.cuda.synchronize()
    kda.check_status()
    return torch.cat(outs, dim=1), final


@pytest.mark.parametrize("cuts", [(64,), (300,), (100, 650), (64, 128, 832), (1, 2, 999)])
def test_split_equals_whole_sequence(cuts):
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=2, H=3, T=1000, seed=7000 + sum(cuts))
    x = I.make_inputs(w, "cuda")
    out, final = _split_run(x, cuts)
    o_ref, s_ref = oracle.forward(*(x[n] for n in NAMES), x["initial_state"])
    assert oracle.parity_error(out.cpu().numpy(), o_ref) <= TOL
    assert oracle.parity_error(final.cpu().numpy(), s_ref) <= TOL
    ws = kda.make_workspace(w.B, w.T, w.H, 128, 128)
    o_w, s_w = kda.forward(*(x[n] for n in NAMES), x["initial_state"], workspace=ws)
    torch.cuda.synchronize()
    assert oracle.parity_error(out.cpu().numpy(), o_w.cpu().double().numpy()) <= 2 * TOL


def test_split_long_context_eight_segments_full_head_chains():
    """B1 H40 (full-head chain kernels), T 16384 in eight segments; sampled heads."""
    w = I.scaled(I.PREFILL_H32_T64K, H=40, T=16384, seed=7100)
    x = I.make_inputs(w, "cuda")
    out, final = _split_run(x, [2048 * i for i in range(1, 8)])
    for h in (0, 33):
        sub = {n: x[n][:, :, h:h + 1].contiguous() for n in NAMES}
        o_ref, s_ref = oracle.forward(*(sub[n] for n in NAMES), None)
        assert oracle.parity_error(out[:, :, h:h + 1].cpu().numpy(), o_ref) <= TOL
        assert oracle.parity_error(final[:, h:h + 1].cpu().numpy(), s_ref) <= TOL


def test_transfer_is_the_state_map_with_zero_values():
    """P S0 = the final state of the segment run from S0 with zero values."""
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=1, H=2, T=200, seed=7200)
    x = I.make_inputs(w, "cuda")
    ws = kda.make_workspace(w.B, w.T, w.H, 128, 128, segment=True)
    _, _, P = kda.segment_local(*(x[n] for n in NAMES), None, workspace=ws)
    z = torch.zeros_like(x["v"])
    _, s_ref = oracle.forward(x["q"], x["k"], z, x["log_alpha"], x["beta"], x["initial_state"])
    got = torch.einsum("bhij,bhjv->bhiv", P.double().cpu(), x["initial_state"].double().cpu()).numpy()
    assert oracle.parity_error(got, s_ref) <= TOL


def test_start_state_fold():
    rng = np.random.default_rng(3)
    R, B, H = 5, 2, 3
    P = (0.1 * rng.standard_normal((R, B, H, 128, 128))).astype(np.float32)
    F = rng.standard_normal((R, B, H, 128, 128)).astype(np.float32)
    ref = F[0].astype(np.float64)
    for j in range(1, R):
        ref = F[j] + np.einsum("bhij,bhjv->bhiv", P[j].astype(np.float64), ref)
    got = kda.segment_start_state(torch.from_numpy(P).cuda(), torch.from_numpy(F).cuda())
    torch.cuda.synchronize()
    assert oracle.parity_error(got.cpu().numpy(), ref) <= 1e-5
