"""Parity on the named workloads at their full sizes, every head and every step.

The benchmark times the long-context prefill (B1 H32 T65536), the batched
prefill with a carried state (B4 H32 T16384) and 1024 sequential decode steps
of B256 H32.  Here the same calls, on the same seeded inputs, are compared
with the fp64 oracle on ALL of their outputs and final states:

* prefill: every (b, h) of every token, through each prefill entry point of
  the C ABI (``kda_forward_ws`` with the fastest workspace, which the
  benchmark times; ``kda_forward`` on its pooled workspace; ``kda_forward_ws``
  with no workspace, the one-kernel prefill; ``kda_forward_noalloc``),
  against one oracle run per workload;
* decode: the output of every one of the 1024 steps for every sequence and
  head, and the state after the last step.  A decode step is one token of the
  recurrence, so the oracle runs each group of sequences through all 1024
  steps as one token sequence (same arithmetic, no state copies between
  steps), while the GPU runs the 1024 in-place ``kda_decode_step`` calls the
  benchmark runs.

Bar (max |gpu - oracle| / rms(oracle), outputs and final states separately):
2e-3 for bf16 inputs.  For decode the bar holds for every step's outputs on
their own rms, not only over the whole run.
"""
import math

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


class _Err:
    """max |gpu - ref| and sum(ref^2) accumulated over slices, so that the
    metric over a multi-GB output never needs a full fp64 copy of both."""

    def __init__(self):
        self.max_abs = 0.0
        self.sumsq = 0.0
        self.n = 0

    def add(self, gpu, ref):
        g = np.asarray(gpu, dtype=np.float64)
        r = np.asarray(ref, dtype=np.float64)
        if r.size == 0:
            return
        self.max_abs = max(self.max_abs, float(np.max(np.abs(g - r))))
        self.sumsq += float(np.sum(r * r))
        self.n += r.size

    def value(self):
        rms = math.sqrt(self.sumsq / self.n) if self.n else 0.0
        return self.max_abs / rms if rms > 0 else self.max_abs


def _prefill_paths(w, x):
    """Outputs and final states of the three prefill entry points on x."""
    res = {}
    ws = kda.make_workspace(w.B, w.T, w.H, w.dk, w.dv)
    assert ws is not None
    res["kda_forward_ws"] = kda.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                        x["initial_state"], workspace=ws)
    torch.cuda.synchronize()
    kda.check_status()
    del ws
    torch.cuda.empty_cache()
    res["kda_forward"] = kda.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["initial_state"])
    res["kda_forward_ws (no workspace: one kernel)"] = kda.forward(
        x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["initial_state"], one_kernel=True)
    res["kda_forward_noalloc"] = kda.forward_noalloc(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                                     x["initial_state"])
    torch.cuda.synchronize()
    kda.check_status()
    return res


def _check_prefill_all_heads(w):
    x = I.make_inputs(w, "cuda")
    res = _prefill_paths(w, x)
    o_ref, s_ref = oracle.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["initial_state"])
    report = {}
    for name, (out, sT) in res.items():
        assert torch.isfinite(sT).all(), name
        eo, es = _Err(), _Err()
        step = 4096
        for t0 in range(0, w.T, step):
            eo.add(out[:, t0:t0 + step].cpu().numpy(), o_ref[:, t0:t0 + step])
        es.add(sT.cpu().numpy(), s_ref)
        report[name] = (eo.value(), es.value())
    for name, (e_o, e_s) in report.items():
        assert e_o <= TOL and e_s <= TOL, "%s: output %.3g, state %.3g (bar %.0e); all: %s" % (
            name, e_o, e_s, TOL, report)
    return report


def test_prefill_h16_t4096_all_heads_every_path():
    _check_prefill_all_heads(I.PREFILL_H16_T4K)


def test_long_context_h32_t65536_all_heads_every_path():
    _check_prefill_all_heads(I.PREFILL_H32_T64K)


def test_batched_carried_state_b4_t16384_all_heads_every_path():
    _check_prefill_all_heads(I.PREFILL_B4_T16K_STATE)


def test_decode_b256_h32_all_1024_steps():
    w = I.DECODE_B256
    x = I.make_inputs(w, "cuda")                      # every step at once: [steps, B, H, d]
    n = x["q"].shape[0]
    assert n == w.steps == 1024
    state = x["initial_state"].clone()
    outs = torch.empty((n, w.B, w.H, w.dv), device="cuda")
    for s in range(n):
        kda.decode_step(x["q"][s], x["k"][s], x["v"][s], x["log_alpha"][s], x["beta"][s], state, out=outs[s])
    torch.cuda.synchronize()
    kda.check_status()
    assert torch.isfinite(outs).all() and torch.isfinite(state).all()

    step_max = np.zeros(n)
    step_sumsq = np.zeros(n)
    es = _Err()
    G = 32                                            # sequences per oracle call
    for b0 in range(0, w.B, G):
        # the group's inputs as token sequences: [G, steps, H, d]
        seq = {nm: x[nm][:, b0:b0 + G].transpose(0, 1).contiguous().cpu() for nm in NAMES}
        o_ref, s_ref = oracle.forward(seq["q"], seq["k"], seq["v"], seq["log_alpha"], seq["beta"],
                                      x["initial_state"][b0:b0 + G])
        o_gpu = outs[:, b0:b0 + G].transpose(0, 1).cpu().numpy().astype(np.float64)
        diff = np.abs(o_gpu - o_ref).reshape(o_ref.shape[0], n, -1)
        step_max = np.maximum(step_max, diff.max(axis=(0, 2)))
        step_sumsq += (o_ref * o_ref).reshape(o_ref.shape[0], n, -1).sum(axis=(0, 2))
        es.add(state[b0:b0 + G].cpu().numpy(), s_ref)
    per_step = step_max / np.sqrt(step_sumsq / (w.B * w.H * w.dv))
    worst = int(np.argmax(per_step))
    assert per_step[worst] <= TOL, "decode step %d: output error %.3g" % (worst, per_step[worst])
    overall = step_max.max() / math.sqrt(step_sumsq.sum() / (n * w.B * w.H * w.dv))
    assert overall <= TOL, "decode outputs over all steps: %.3g" % overall
    assert es.value() <= TOL, "state after %d steps: %.3g" % (n, es.value())
