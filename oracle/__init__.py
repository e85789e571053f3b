"""CPU oracle for the Kimi Delta Attention (KDA) forward pass.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline / reference leg may import this package.  The library's product
path never calls it, and it shares no code with the CUDA path.

Two implementations of the same definition, both fp64 on the exact input
values: the KDA recurrence per head and token t,

    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
    o_t = scale * S_t^T q_t,

the per-channel decay and beta-scaled delta rule of "Kimi Delta Attention: The
Linear Attention Behind Kimi K2 and Qwen3" (§TL;DR; the order of the operations
is stated in prose in §How Kimi Delta Attention works step by step) with the
forgetting factor (I - beta k k^T) of "KDA Technical Deep Dive", §From attention
to recurrent state.  Both evaluate the product in its expanded form, decay,
then the delta-rule error beta_t (v_t - S~^T k_t), then S_t = S~ + k_t e^T,
then the read with the 1/sqrt(d_k)-scaled query:

* ``forward``     -- plain C (``kda_oracle.c``), threaded over heads; used for
                     parity at realistic sizes and for the timed CPU baseline.
* ``forward_np``  -- plain numpy, a loop over tokens vectorised over (B, H);
                     used for small cases and to cross-check ``forward``.
* ``gdn_forward`` -- the scalar-gate variants (Gated DeltaNet, DeltaNet) as
                     ``forward`` with the gate repeated over key channels.
* ``forward_raw`` -- raw activations: sigmoid gate pre-activations and
                     unnormalised q, k, prepared in fp64, then ``forward``.
* ``backward``    -- gradients of the forward with respect to every input, by
                     reverse-mode automatic differentiation (torch.autograd, CPU,
                     fp64) of the same token recurrence.

Both store the state as ``[B, H, dk, dv]`` (the transpose of the pages'
(d_v, d_k) key-to-value map), so the per-channel decay scales rows and the
prediction for a key k is ``S^T k`` here.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``kda_oracle.c`` into ``libkda_oracle.so`` next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        f = lib.kda_oracle_forward
        f.restype = ctypes.c_int
        f.argtypes = [ctypes.c_void_p] * 8 + [ctypes.c_int] * 5 + [ctypes.c_double, ctypes.c_int]
        lib.kda_oracle_default_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def default_threads() -> int:
    return int(_load().kda_oracle_default_threads())


def _as_f32(x) -> np.ndarray:
    """Exact fp32 copy of a torch tensor (bf16 or fp32) or array."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def _as_f64(x) -> Optional[np.ndarray]:
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def forward(q, k, v, log_alpha, beta, initial_state=None, scale=None, nthreads=0):
    """fp64 KDA forward by the token recurrence (C implementation).

    Arguments are torch tensors or numpy arrays in the library layout:
    q, k, log_alpha ``[B,T,H,dk]``; v ``[B,T,H,dv]``; beta ``[B,T,H]``;
    initial_state ``[B,H,dk,dv]`` or None (zeros).  ``scale`` defaults to
    ``1/sqrt(dk)``.  Returns ``(out [B,T,H,dv], final_state [B,H,dk,dv])`` as
    fp64 numpy arrays.
    """
    qf, kf, vf, af, bf = (_as_f32(x) for x in (q, k, v, log_alpha, beta))
    B, T, H, dk = qf.shape
    dv = vf.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(dk)
    s0 = _as_f64(initial_state)
    out = np.empty((B, T, H, dv), dtype=np.float64)
    sT = np.empty((B, H, dk, dv), dtype=np.float64)
    rc = _load().kda_oracle_forward(_ptr(qf), _ptr(kf), _ptr(vf), _ptr(af), _ptr(bf),
                                    _ptr(s0), _ptr(out), _ptr(sT),
                                    B, T, H, dk, dv, float(scale), int(nthreads))
    if rc != 0:
        raise RuntimeError("kda_oracle_forward failed with code %d" % rc)
    return out, sT


def forward_np(q, k, v, log_alpha, beta, initial_state=None, scale=None, exact64=False):
    """fp64 KDA forward by the token recurrence (numpy implementation).

    Same arguments and results as :func:`forward`.  Meant for small inputs.
    ``exact64`` takes fp64 inputs as they are instead of as their fp32 values
    (finite differences of the forward need perturbations below fp32 spacing).
    """
    conv = _as_f64 if exact64 else (lambda x: _as_f32(x).astype(np.float64))
    qf, kf, vf, af, bf = (conv(x) for x in (q, k, v, log_alpha, beta))
    B, T, H, dk = qf.shape
    dv = vf.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(dk)
    S = np.zeros((B, H, dk, dv)) if initial_state is None else _as_f64(initial_state).copy()
    out = np.empty((B, T, H, dv))
    for t in range(T):
        alpha = np.exp(af[:, t])                           # [B,H,dk]
        S = S * alpha[..., :, None]                        # decay rows (key channels)
        p = np.einsum("bhcx,bhc->bhx", S, kf[:, t])        # S~^T k
        e = bf[:, t, :, None] * (vf[:, t] - p)             # beta (v - p)
        S = S + kf[:, t][..., :, None] * e[..., None, :]   # S~ + k e^T
        out[:, t] = scale * np.einsum("bhcx,bhc->bhx", S, qf[:, t])
    return out, S


def gdn_forward(q, k, v, log_alpha, beta, initial_state=None, scale=None, nthreads=0):
    """fp64 forward of the scalar-gate members of the family.

    Gated DeltaNet decays every key channel of the state by the same alpha_t;
    KDA's gate is the per-channel refinement of it ("Kimi Delta Attention: The
    Linear Attention Behind Kimi K2 and Qwen3", §DeltaNet, Gated DeltaNet, and
    KDA, comparison table).  DeltaNet has no decay (alpha = 1; "KDA Technical
    Deep Dive", §From attention to recurrent state (delta rule)).  So this is
    :func:`forward` with ``log_alpha [B,T,H]`` repeated over the dk key
    channels, or zeros when ``log_alpha`` is None.
    """
    qf = _as_f32(q)
    B, T, H, dk = qf.shape
    if log_alpha is None:
        la = np.zeros((B, T, H, dk), dtype=np.float32)
    else:
        g = _as_f32(log_alpha)
        if g.shape != (B, T, H):
            raise ValueError("log_alpha has shape %s, expected %s" % (g.shape, (B, T, H)))
        la = np.ascontiguousarray(np.repeat(g[..., None], dk, axis=-1))
    return forward(qf, k, v, la, beta, initial_state, scale=scale, nthreads=nthreads)


def forward_raw(q, k, v, gate, beta, initial_state=None, logsigmoid_gate=True, normalize_qk=True,
                scale=None, nthreads=0):
    """fp64 forward of raw layer activations: the steps before the path, then :func:`forward`.

    With ``logsigmoid_gate`` the gate holds pre-activations x of the sigmoid
    retention gate ("KDA Technical Deep Dive", §How the Kimi gate changes
    memory: alpha a sigmoid-like value in (0, 1)), so log alpha = log(sigmoid(x))
    = -log(1 + e^{-x}).  With ``normalize_qk`` q and k are divided by the L2 norm
    of their dk channels per (b, t, h) (the normalised keys the KDA page says the
    path receives); a zero row stays zero.  Both in fp64 on the exact inputs.
    """
    q64, k64, g64 = (_as_f64(x) for x in (q, k, gate))
    if normalize_qk:
        def unit(x):
            n = np.linalg.norm(x, axis=-1, keepdims=True)
            return np.where(n > 0, x / np.where(n > 0, n, 1.0), 0.0)
        q64, k64 = unit(q64), unit(k64)
    la = -np.logaddexp(0.0, -g64) if logsigmoid_gate else g64
    return forward(q64, k64, v, la, beta, initial_state, scale=scale, nthreads=nthreads)


def backward(q, k, v, log_alpha, beta, d_out, initial_state=None, d_final_state=None, scale=None,
             segment=64):
    """fp64 gradients of the KDA forward with respect to every input.

    The loss is L = sum(O * d_out) + sum(S_T * d_final_state): ``d_out`` [B,T,H,dv]
    and ``d_final_state`` [B,H,dk,dv] (None: zeros) are the cotangents of the
    outputs and of the final state.  The gradient is the derivative of the token
    recurrence of "Kimi Delta Attention: The Linear Attention Behind Kimi K2 and
    Qwen3", §How Kimi Delta Attention works step by step (the same steps as
    :func:`forward_np`, written in torch ops), taken by torch.autograd in fp64 on
    the exact input values.  The pages give no gradient formulas ("KDA Technical
    Deep Dive", §Systems and implementation tradeoffs, Training, names only
    chunkwise training), so the definition is the derivative itself.  Tokens run in
    segments of ``segment`` whose states are recomputed during the backward sweep
    (torch.utils.checkpoint), so memory grows with T / segment.

    Returns a dict of fp64 numpy arrays: ``dq``, ``dk``, ``dv``, ``dlog_alpha``,
    ``dbeta`` (shapes of the inputs) and ``dinitial_state`` [B,H,dk,dv] (the
    gradient with respect to the initial state; a zero state when it is None).
    """
    import torch
    from torch.utils.checkpoint import checkpoint

    def exact(x):
        return torch.from_numpy(_as_f32(x).astype(np.float64))

    qt, kt, vt, at, bt = (exact(x).requires_grad_(True) for x in (q, k, v, log_alpha, beta))
    B, T, H, dk = qt.shape
    dv = vt.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(dk)
    s0 = (torch.zeros((B, H, dk, dv), dtype=torch.float64) if initial_state is None
          else torch.from_numpy(_as_f64(initial_state)).clone())
    s0.requires_grad_(True)
    d_o = torch.from_numpy(_as_f64(d_out))
    d_s = (torch.zeros((B, H, dk, dv), dtype=torch.float64) if d_final_state is None
           else torch.from_numpy(_as_f64(d_final_state)))

    def run(S, q_, k_, v_, a_, b_):
        outs = []
        for t in range(q_.shape[1]):
            S = S * torch.exp(a_[:, t]).unsqueeze(-1)                   # decay rows (key channels)
            p = torch.einsum("bhcx,bhc->bhx", S, k_[:, t])               # S~^T k
            e = b_[:, t].unsqueeze(-1) * (v_[:, t] - p)                  # beta (v - p)
            S = S + k_[:, t].unsqueeze(-1) * e.unsqueeze(-2)             # S~ + k e^T
            outs.append(scale * torch.einsum("bhcx,bhc->bhx", S, q_[:, t]))
        return S, torch.stack(outs, 1)

    S = s0
    loss = torch.zeros((), dtype=torch.float64)
    for t0 in range(0, T, segment):
        sl = slice(t0, min(T, t0 + segment))
        S, O = checkpoint(run, S, qt[:, sl], kt[:, sl], vt[:, sl], at[:, sl], bt[:, sl], use_reentrant=False)
        loss = loss + (O * d_o[:, sl]).sum()
    loss = loss + (S * d_s).sum()
    g = torch.autograd.grad(loss, [qt, kt, vt, at, bt, s0], allow_unused=True)
    names = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dinitial_state")
    ref = (qt, kt, vt, at, bt, s0)
    return {n: (gi if gi is not None else torch.zeros_like(r)).detach().numpy() for n, gi, r in zip(names, g, ref)}


def parity_error(x_gpu, x_ref) -> float:
    """max |x_gpu - x_ref| / rms(x_ref), the parity metric for outputs and states."""
    g = np.asarray(x_gpu, dtype=np.float64)
    r = np.asarray(x_ref, dtype=np.float64)
    if r.size == 0:
        return 0.0
    rms = math.sqrt(float(np.mean(r * r)))
    err = float(np.max(np.abs(g - r)))
    if rms == 0.0:
        return err
    return err / rms
