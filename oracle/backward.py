"""Reverse mode of the KDA recurrence -- TEST INFRASTRUCTURE (part of the oracle).

Gradients of a loss through the token recurrence ("Kimi Linear: An Expressive,
Efficient Attention Architecture", section Method, "From Linear Attention to
KDA": S~ = Diag(alpha_t) S_{t-1}, S_t = S~ + beta_t k_t (v_t - S~^T k_t)^T,
o_t = S_t^T q_t; alpha = exp(g)), written out step by step in fp64.  Training
the layer (section "Training and Inference": training runs the chunk form)
needs dq, dk, dv, dg, dbeta and the initial-state gradient given do and the
gradient of the final state.

Forward, per token (scale multiplies q):
    S~ = Diag(a) S_prev,  y = S~^T k,  u = beta (v - y),  S = S~ + k u^T,  o = S^T (scale q).
Reverse, from t = T down to 1, with G the running gradient of S_t:
    G += (scale q) do^T;             dq = scale S do
    du = G^T k;  dk = G u;           dv = beta du;  dbeta = du . (v - y);  dy = -beta du
    G~ = G + k dy^T;  dk += S~ dy;   dg = rowsum(G~ (.) S~)   (d a = rowsum(G~ (.) S_prev), a = e^g)
    G  <- Diag(a) G~                 (the gradient of S_{t-1})
and the initial-state gradient is the final G.  Every line is the chain rule of
the forward line it inverts; nothing is fused or reordered.
"""
from __future__ import annotations

import numpy as np


def kda_recurrent_backward(q, k, v, g, beta, do, s0=None, ds_final=None, scale=1.0):
    """One sequence or a batch: q, k, v, g, do [B,T,H,D] (or [T,H,D]); beta [B,T,H].

    Returns dq, dk, dv, dg (same shapes), dbeta [B,T,H] and ds0 [B,H,D,D]."""
    q, k, v, g, beta, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta, do))
    squeeze = q.ndim == 3
    if squeeze:
        q, k, v, g, beta, do = (x[None] for x in (q, k, v, g, beta, do))
    B, T, H, D = q.shape
    DV = v.shape[3]
    S0 = np.zeros((B, H, D, DV)) if s0 is None else np.asarray(s0, dtype=np.float64).reshape(B, H, D, DV)
    G0 = np.zeros((B, H, D, DV)) if ds_final is None else np.asarray(ds_final, dtype=np.float64).reshape(B, H, D, DV)
    dq, dk, dv, dg = (np.zeros_like(x) for x in (q, k, v, g))
    dbeta = np.zeros_like(beta)
    ds0 = np.zeros((B, H, D, DV))
    for b in range(B):
        for h in range(H):
            # forward, keeping every S_{t-1}
            S = S0[b, h].copy()
            prev = []
            for t in range(T):
                prev.append(S)
                a = np.exp(g[b, t, h])
                St = a[:, None] * S
                y = St.T @ k[b, t, h]
                u = beta[b, t, h] * (v[b, t, h] - y)
                S = St + np.outer(k[b, t, h], u)
            # reverse
            G = G0[b, h].copy()
            for t in range(T - 1, -1, -1):
                Sp = prev[t]
                a = np.exp(g[b, t, h])
                kt, qt, vt, bt, dot = k[b, t, h], scale * q[b, t, h], v[b, t, h], beta[b, t, h], do[b, t, h]
                St = a[:, None] * Sp
                y = St.T @ kt
                u = bt * (vt - y)
                S = St + np.outer(kt, u)
                G = G + np.outer(qt, dot)
                dq[b, t, h] = scale * (S @ dot)
                du = G.T @ kt
                dkt = G @ u
                dv[b, t, h] = bt * du
                dbeta[b, t, h] = du @ (vt - y)
                dy = -bt * du
                Gt = G + np.outer(kt, dy)
                dkt = dkt + St @ dy
                dk[b, t, h] = dkt
                dg[b, t, h] = (Gt * St).sum(axis=1)
                G = a[:, None] * Gt
            ds0[b, h] = G
    if squeeze:
        dq, dk, dv, dg, dbeta = (x[0] for x in (dq, dk, dv, dg, dbeta))
    return dq, dk, dv, dg, dbeta, ds0
