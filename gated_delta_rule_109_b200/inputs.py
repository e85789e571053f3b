"""Seeded synthetic inputs for the KDA forward workloads.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests. It holds only random draws and the input preconditions the
callers of a KDA layer are expected to meet; it holds none of the KDA
recurrence itself.

Input recipe (one draw order for every workload, from one seeded
``torch.Generator`` on the requested device):

1. ``q``  ~ N(0, 1), L2-normalised per token in fp32, then cast to the input
   dtype.  Keys and queries arriving normalised is the precondition stated in
   "Kimi Delta Attention: The Linear Attention Behind Kimi K2 and Qwen3",
   §Impact and analysis (warning box) and FAQ "Why does DeltaNet need keys to
   be normalized?".
2. ``k``  ~ N(0, 1), normalised and cast the same way.
3. ``v``  ~ N(0, 1), cast to the input dtype.
4. ``x_alpha`` ~ N(mu_a, sd_a); ``log_alpha = logsigmoid(x_alpha)`` computed in
   fp64 and rounded once to fp32.  A sigmoid retention gate in (0, 1) is the
   parameterisation named in "KDA Technical Deep Dive", §How the Kimi gate
   changes memory.
5. ``x_beta``  ~ N(mu_b, sd_b); ``beta = sigmoid(x_beta)`` in fp32.
6. ``S_0`` ~ N(0, sd_s) in fp32 when the workload carries a state, else absent.

Raw-activation variant (``make_raw_inputs``, for the fused steps before the
path): the same draws with q and k cast to the input dtype without
normalisation, and the gate returned as its pre-activation ``x_alpha``
(fp32) instead of ``logsigmoid(x_alpha)``.

Shapes follow the library's layout: q, k ``[B, T, H, dk]``; v ``[B, T, H, dv]``;
log_alpha ``[B, T, H, dk]`` fp32; beta ``[B, T, H]`` fp32; state
``[B, H, dk, dv]`` fp32.  Decode workloads draw every step at once with a
leading ``steps`` axis: ``[steps, B, H, d]``.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic KDA workload: sizes, input distributions and seed."""

    name: str
    B: int
    H: int
    T: int            # sequence length for prefill; 1 for a decode step
    dk: int
    dv: int
    dtype: str        # "f32" or "bf16": dtype of q, k, v
    alpha_mu: float
    alpha_sd: float
    beta_mu: float
    beta_sd: float
    state_sd: Optional[float]   # None: zero initial state (no buffer passed)
    seed: int
    steps: int = 0    # decode only: number of sequential single-token steps
    final_state: bool = True

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def is_decode(self) -> bool:
        return self.steps > 0


# The five workloads the library is specified and measured on.
TINY_F32 = Workload("tiny_f32_b1_h2_t256_d64", 1, 2, 256, 64, 64, "f32",
                    3.0, 1.0, 0.0, 1.0, None, 0)
PREFILL_H16_T4K = Workload("prefill_bf16_b1_h16_t4096_d128", 1, 16, 4096, 128, 128,
                           "bf16", 4.0, 1.0, 0.0, 1.0, None, 1)
PREFILL_H32_T64K = Workload("prefill_bf16_b1_h32_t65536_d128", 1, 32, 65536, 128, 128,
                            "bf16", 4.0, 1.0, 0.0, 1.0, None, 2)
PREFILL_B4_T16K_STATE = Workload("prefill_bf16_b4_h32_t16384_d128_state", 4, 32, 16384,
                                 128, 128, "bf16", 2.0, 1.5, 0.5, 1.0, 0.02, 3)
DECODE_B256 = Workload("decode_bf16_b256_h32_d128_1024steps", 256, 32, 1, 128, 128,
                       "bf16", 4.0, 1.0, 0.0, 1.0, 0.02, 4, steps=1024)

WORKLOADS = [TINY_F32, PREFILL_H16_T4K, PREFILL_H32_T64K, PREFILL_B4_T16K_STATE, DECODE_B256]


def scaled(w: Workload, **changes) -> Workload:
    """A copy of ``w`` with some fields replaced (smaller sizes for tests)."""
    return dataclasses.replace(w, **changes)


def _normal(shape, gen, device, mu=0.0, sd=1.0):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if sd != 1.0:
        x.mul_(sd)
    if mu != 0.0:
        x.add_(mu)
    return x


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def make_inputs(w: Workload, device="cpu", steps: Optional[int] = None) -> dict:
    """Draw the workload's inputs on ``device``.

    Returns a dict with ``q, k, v, log_alpha, beta`` and ``initial_state``
    (``None`` for a zero state).  For decode workloads every tensor has a
    leading axis of ``steps`` (default ``w.steps``) and no T axis.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    if w.is_decode:
        n = w.steps if steps is None else steps
        lead = (n, w.B, w.H)
    else:
        lead = (w.B, w.T, w.H)
    dt = w.torch_dtype
    q = _unit_rows(_normal(lead + (w.dk,), gen, device)).to(dt)
    k = _unit_rows(_normal(lead + (w.dk,), gen, device)).to(dt)
    v = _normal(lead + (w.dv,), gen, device).to(dt)
    xa = _normal(lead + (w.dk,), gen, device, w.alpha_mu, w.alpha_sd)
    log_alpha = torch.nn.functional.logsigmoid(xa.double()).float()
    del xa
    xb = _normal(lead, gen, device, w.beta_mu, w.beta_sd)
    beta = torch.sigmoid(xb)
    del xb
    s0 = None
    if w.state_sd is not None:
        s0 = _normal((w.B, w.H, w.dk, w.dv), gen, device, 0.0, w.state_sd)
    return dict(q=q.contiguous(), k=k.contiguous(), v=v.contiguous(),
                log_alpha=log_alpha.contiguous(), beta=beta.contiguous(),
                initial_state=s0)


def make_raw_inputs(w: Workload, device="cpu") -> dict:
    """The draws of :func:`make_inputs` before the steps the prefill can fuse: q, k
    cast to the input dtype without L2 normalisation, and ``gate`` = the gate
    pre-activations x_alpha (fp32).  Prefill workloads only."""
    if w.is_decode:
        raise ValueError("prefill workloads only")
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    lead = (w.B, w.T, w.H)
    dt = w.torch_dtype
    q = _normal(lead + (w.dk,), gen, device).to(dt)
    k = _normal(lead + (w.dk,), gen, device).to(dt)
    v = _normal(lead + (w.dv,), gen, device).to(dt)
    xa = _normal(lead + (w.dk,), gen, device, w.alpha_mu, w.alpha_sd)
    xb = _normal(lead, gen, device, w.beta_mu, w.beta_sd)
    beta = torch.sigmoid(xb)
    del xb
    s0 = None
    if w.state_sd is not None:
        s0 = _normal((w.B, w.H, w.dk, w.dv), gen, device, 0.0, w.state_sd)
    return dict(q=q.contiguous(), k=k.contiguous(), v=v.contiguous(), gate=xa.contiguous(),
                beta=beta.contiguous(), initial_state=s0)
