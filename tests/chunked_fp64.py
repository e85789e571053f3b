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


def _chunk_terms(kk, qq, vv, bb, la, S, scale, mm=np.matmul):
    """The chunk's forward quantities (module docstring) for entering state S; every
    matrix product goes through ``mm``."""
    c = kk.shape[0]
    G = np.cumsum(la, axis=0)
    eG, emG, eL = np.exp(G), np.exp(-G), np.exp(G[-1] - G)
    Kt, Kb, Qt, Kh = kk * eG, kk * emG, scale * qq * eG, kk * eL
    P = np.tril(mm(Kt, Kb.T), -1)
    A = bb[:, None] * P
    M = np.tril(mm(Qt, Kb.T))
    Tm = np.linalg.inv(np.eye(c) + A)
    W = mm(Tm, bb[:, None] * Kt)
    U = mm(Tm, bb[:, None] * vv)
    D = U - mm(W, S)
    gam = np.exp(G[-1])
    return dict(G=G, eG=eG, emG=emG, eL=eL, Kt=Kt, Kb=Kb, Qt=Qt, Kh=Kh, P=P, M=M, Tm=Tm, W=W, D=D,
                gam=gam, S_next=gam[:, None] * S + mm(Kh.T, D))


def chunked_backward(q, k, v, log_alpha, beta, d_out, initial_state=None, d_final_state=None,
                     scale=None, C=64, mm=np.matmul):
    """Reverse-mode derivative of the chunk algebra above, one chunk at a time.

    The loss is L = sum(O * d_out) + sum(S_T * d_final_state).  A forward sweep keeps
    the state entering every chunk; a backward sweep carries dS = dL/dS (the state
    leaving the chunk) from the last chunk to the first.  Per chunk, with the
    forward quantities recomputed from its entering state S:

      serial (the transpose of the forward chain: two dependent products per chunk)
        dD    = M^T dO + Kh dS
        dS_in = Diag(Gam) dS + Qt^T dO - W^T dD
      chunk-parallel, given S, dS and dD
        dM  = L o (dO D^T)             dQt = dO S^T + dM Kb        dKb = dM^T Qt
        dKh = D dS^T                   dGam = rowsum(dS o S)
        dW  = -dD S^T                  dU = dD
        dTm = dU (Diag(beta) V)^T + dW (Diag(beta) Kt)^T
        dA  = -(Tm^T dTm Tm^T) o strictly_lower
        dv  = Diag(beta) Tm^T dU       dKt = Diag(beta) (Tm^T dW + dA Kb)    dKb += (Diag(beta) dA)^T Kt
        dbeta = rowsum(Tm^T dU o V) + rowsum(Tm^T dW o Kt) + rowsum(dA o P)
      and through the exponentials (Kt = k e^G, Kb = k e^-G, Qt = scale q e^G,
      Kh = k e^{G_last - G}, Gam = e^{G_last}) to dk, dq and dG, whose suffix sums
      over the chunk are dlog_alpha (G is an inclusive prefix sum).

    Every matrix product goes through ``mm`` (a test passes a model of a kernel's
    product precision).  Returns the dict of oracle.backward: dq, dk, dv, dlog_alpha,
    dbeta, dinitial_state.
    """
    q, k, v, la, be, g_o = (np.asarray(x, dtype=np.float64) for x in (q, k, v, log_alpha, beta, d_out))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(dk)
    S0 = (np.zeros((B, H, dk, dv)) if initial_state is None
          else np.asarray(initial_state, dtype=np.float64))
    gS = (np.zeros((B, H, dk, dv)) if d_final_state is None
          else np.asarray(d_final_state, dtype=np.float64))
    res = {n: np.zeros(x.shape) for n, x in (("dq", q), ("dk", k), ("dv", v), ("dlog_alpha", la),
                                             ("dbeta", be))}
    res["dinitial_state"] = np.zeros((B, H, dk, dv))
    starts = list(range(0, T, C))
    for b in range(B):
        for h in range(H):
            sl = lambda x, s: x[b, s:min(T, s + C), h]
            S_in, S = [], S0[b, h].copy()
            for s in starts:
                S_in.append(S)
                S = _chunk_terms(sl(k, s), sl(q, s), sl(v, s), sl(be, s), sl(la, s), S, scale, mm)["S_next"]
            dS = gS[b, h].copy()
            for s, S in zip(reversed(starts), reversed(S_in)):
                kk, qq, vv, bb, dO = sl(k, s), sl(q, s), sl(v, s), sl(be, s), sl(g_o, s)
                f = _chunk_terms(kk, qq, vv, bb, sl(la, s), S, scale, mm)
                c = kk.shape[0]
                dD = mm(f["M"].T, dO) + mm(f["Kh"], dS)
                dS_in = f["gam"][:, None] * dS + mm(f["Qt"].T, dO) - mm(f["W"].T, dD)
                dM = np.tril(mm(dO, f["D"].T))
                dQt = mm(dO, S.T) + mm(dM, f["Kb"])
                dKb = mm(dM.T, f["Qt"])
                dKh = mm(f["D"], dS.T)
                dGam = (dS * S).sum(axis=1)
                dW = -mm(dD, S.T)
                Yv, Yk = bb[:, None] * vv, bb[:, None] * f["Kt"]
                dTm = mm(dD, Yv.T) + mm(dW, Yk.T)
                dYv, dYk = mm(f["Tm"].T, dD), mm(f["Tm"].T, dW)
                dA = -np.tril(mm(mm(f["Tm"].T, dTm), f["Tm"].T), -1)
                dP = bb[:, None] * dA
                dKt = bb[:, None] * dYk + mm(dP, f["Kb"])
                dKb = dKb + mm(dP.T, f["Kt"])
                e = s + c
                res["dv"][b, s:e, h] = bb[:, None] * dYv
                res["dbeta"][b, s:e, h] = ((dYv * vv).sum(1) + (dYk * f["Kt"]).sum(1)
                                           + (dA * f["P"]).sum(1))
                res["dk"][b, s:e, h] = dKt * f["eG"] + dKb * f["emG"] + dKh * f["eL"]
                res["dq"][b, s:e, h] = scale * dQt * f["eG"]
                dG = dKt * f["Kt"] - dKb * f["Kb"] + dQt * f["Qt"] - dKh * f["Kh"]
                dG[-1] += (dKh * f["Kh"]).sum(axis=0) + dGam * f["gam"]
                res["dlog_alpha"][b, s:e, h] = np.cumsum(dG[::-1], axis=0)[::-1]
                dS = dS_in
            res["dinitial_state"][b, h] = dS
    return res
