"""fp64 numpy statement of the chunkwise (WY / UT) form of the KDA forward.

Test helper, not the oracle.  The pages say KDA runs "chunkwise" in production
and that the state at a chunk boundary is the initial condition of the next
chunk ("Kimi Delta Attention: The Linear Attention Behind Kimi K2 and Qwen3",
§How Kimi Delta Attention works step by step; "KDA Technical Deep Dive",
§Systems and implementation tradeoffs, Training) but give no chunk algebra.
This file writes out the re-association of the token recurrence that the CUDA
prefill kernels use, so that a test can check the algebra against the
recurrence in fp64 before any kernel relies on it.

Per (b, h) and chunk of c <= C tokens with entering state S (dk x dv):

  G_t  = sum_{s <= t} log_alpha_s          (inclusive, reset every chunk)
  Kt_t = k_t * exp(G_t)          Kb_t = k_t * exp(-G_t)
  Qt_t = scale * q_t * exp(G_t)  Kh_t = k_t * exp(G_last - G_t)
  A    = Diag(beta) * strictly_lower(Kt Kb^T)         (A_ij = beta_i k_i.(Gam_i/Gam_j) k_j)
  M    = lower_including_diagonal(Qt Kb^T)
  Tm   = (I + A)^-1
  W    = Tm Diag(beta) Kt          U = Tm Diag(beta) V
  D    = U - W S                   (row t is the error e_t of the token step)
  O    = Qt S + M D
  S   <- Diag(exp(G_last)) S + Kh^T D
"""
from __future__ import annotations

import math

import numpy as np


def chunked_forward(q, k, v, log_alpha, beta, initial_state=None, scale=None, C=64):
    q, k, v, la, be = (np.asarray(x, dtype=np.float64) for x in (q, k, v, log_alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(dk)
    S_all = (np.zeros((B, H, dk, dv)) if initial_state is None
             else np.array(initial_state, dtype=np.float64))
    out = np.zeros((B, T, H, dv))
    for b in range(B):
        for h in range(H):
            S = S_all[b, h].copy()
            for s in range(0, T, C):
                e = min(T, s + C)
                c = e - s
                kk, qq, vv = k[b, s:e, h], q[b, s:e, h], v[b, s:e, h]
                bb = be[b, s:e, h]
                G = np.cumsum(la[b, s:e, h], axis=0)
                Kt = kk * np.exp(G)
                Kb = kk * np.exp(-G)
                Qt = scale * qq * np.exp(G)
                Kh = kk * np.exp(G[-1] - G)
                A = bb[:, None] * np.tril(Kt @ Kb.T, -1)
                M = np.tril(Qt @ Kb.T)
                Tm = np.linalg.inv(np.eye(c) + A)
                W = Tm @ (bb[:, None] * Kt)
                U = Tm @ (bb[:, None] * vv)
                D = U - W @ S
                out[b, s:e, h] = Qt @ S + M @ D
                S = np.exp(G[-1])[:, None] * S + Kh.T @ D
            S_all[b, h] = S
    return out, S_all
