"""Reverse mode of the chunkwise KDA form -- TEST INFRASTRUCTURE (part of the oracle).

"Kimi Linear: An Expressive, Efficient Attention Architecture" (research notes),
section "Training and Inference": training runs the chunkwise form; section
"Chunkwise Algorithm" gives its per-chunk pieces (gated gram matrices, the WY
representation, the UT transform, the state carried between chunks).  This module
is the chain rule of that form, chunk by chunk, in fp64 numpy: what a chunked
backward kernel computes, written plainly so that it can be checked by eye against
the forward in ``chunkwise.py`` and, numerically, against the token-by-token
reverse mode in ``backward.py``.

Forward of one chunk (rows r = 0..L-1, entering state S, q already scaled):

  b = cumsum(g)  (per channel);  E[r,i,c] = exp(b[r,c] - b[i,c]) for i <= r, else 0
  M_kk[r,i] = sum_c k[r,c] k[i,c] E[r,i,c];   M_qk[r,i] = sum_c q[r,c] k[i,c] E[r,i,c]
  A = diag(beta) M_kk (strictly lower);  P = M_qk (lower incl. diagonal);  T = (I + A)^{-1}
  X_v = diag(beta) V;  X_k = diag(beta) (K (.) exp(b));  U = T X_v;  W = T X_k
  U~ = U - W S
  O = (Q (.) exp(b)) S + P U~
  S_next = Diag(exp(b_L-1)) S + (K (.) exp(b_L-1 - b))^T U~

Reverse, given dO and dS_next (each line inverts one forward line):

  dS = Diag(exp(b_L-1)) dS_next + (Q (.) exp(b))^T dO - W^T dU~
  dU~ = (K (.) exp(b_L-1 - b)) dS_next + P^T dO;   dP = (dO U~^T) (.) lower
  dU = dU~;  dW = -dU~ S^T;  dT = dU X_v^T + dW X_k^T
  dX_v = T^T dU;  dX_k = T^T dW;  dV = diag(beta) dX_v
  dA = -(T^T dT T^T) (.) strictly lower          (d of the inverse)
  dbeta = rowsum(V (.) dX_v) + rowsum((K (.) exp(b)) (.) dX_k) + rowsum(dA (.) M_kk)
  dM_kk = diag(beta) dA;  dM_qk = dP
  then through the grams (x = k or q in the row role, k in the column role):
  dx[r,c] += sum_i dM[r,i] k[i,c] E[r,i,c];  dk[i,c] += sum_r dM[r,i] x[r,c] E[r,i,c]
  db[r,c] += sum_i dM[r,i] x[r,c] k[i,c] E[r,i,c];  db[i,c] -= the same sum over r
  and through the gated copies of q and k and the chunk-end factors:
  exp(b) (.) Q, exp(b) (.) K:  d(.) (.) exp(b) into dq / dk, d(.) (.) value into db;
  exp(b_L-1 - b) (.) K:  into dk, minus into db_r, plus the column sum into db_L-1;
  exp(b_L-1) on S:  rowsum(S (.) dS_next) (.) exp(b_L-1) into db_L-1
  dg = reverse cumulative sum of db over the chunk's rows.

The state entering each chunk comes from a forward pass over the chunks; the
chunks are then reversed, each handing its dS to the chunk before it.
"""
from __future__ import annotations

import numpy as np

from .chunkwise import unit_lower_inverse


def _chunk_backward(S, q, k, v, g, beta, do, dS_next):
    """One chunk; q is already scaled.  Returns dq, dk, dv, dg, dbeta, dS."""
    L = q.shape[0]
    b = np.cumsum(g, axis=0)                              # [L, DK]
    gam = np.exp(b)
    bL = b[L - 1]
    lower = np.tril(np.ones((L, L)), 0)
    lower_strict = np.tril(np.ones((L, L)), -1)
    diff = b[:, None, :] - b[None, :, :]                  # [r, i, c]
    E = np.exp(np.where(lower[:, :, None] > 0, diff, 0.0)) * lower[:, :, None]
    Mkk = np.einsum("rc,ic,ric->ri", k, k, E)
    Mqk = np.einsum("rc,ic,ric->ri", q, k, E)
    A = beta[:, None] * Mkk * lower_strict
    P = Mqk * lower
    T = unit_lower_inverse(A)
    Kg = k * gam
    Xv = beta[:, None] * v
    Xk = beta[:, None] * Kg
    U = T @ Xv
    W = T @ Xk
    Ut = U - W @ S
    Qg = q * gam
    fL = np.exp(bL[None, :] - b)
    Kd = k * fL
    GL = np.exp(bL)

    # S_next = Diag(GL) S + Kd^T Ut
    dS = GL[:, None] * dS_next
    dKd = Ut @ dS_next.T
    dUt = Kd @ dS_next
    dGL = np.sum(S * dS_next, axis=1)
    # O = Qg S + P Ut
    dQg = do @ S.T
    dS += Qg.T @ do
    dP = (do @ Ut.T) * lower
    dUt += P.T @ do
    # Ut = U - W S
    dU = dUt
    dW = -dUt @ S.T
    dS -= W.T @ dUt
    # U = T Xv, W = T Xk
    dT = dU @ Xv.T + dW @ Xk.T
    dXv = T.T @ dU
    dXk = T.T @ dW
    dv = beta[:, None] * dXv
    dbeta = np.sum(v * dXv, axis=1) + np.sum(Kg * dXk, axis=1)
    dKg = beta[:, None] * dXk
    # T = (I + A)^{-1}, A = diag(beta) Mkk strictly lower
    dA = -(T.T @ dT @ T.T) * lower_strict
    dbeta += np.sum(dA * Mkk, axis=1)
    dMkk = beta[:, None] * dA
    dMqk = dP
    # the gated grams
    dk = np.einsum("ri,ic,ric->rc", dMkk, k, E) + np.einsum("ri,rc,ric->ic", dMkk, k, E)
    dq = np.einsum("ri,ic,ric->rc", dMqk, k, E)
    dk += np.einsum("ri,rc,ric->ic", dMqk, q, E)
    terms = np.einsum("ri,rc,ic,ric->ric", dMkk, k, k, E) + np.einsum("ri,rc,ic,ric->ric", dMqk, q, k, E)
    db = terms.sum(axis=1) - terms.sum(axis=0)
    # gated copies and chunk-end factors
    dq += dQg * gam
    db += dQg * Qg
    dk += dKg * gam
    db += dKg * Kg
    dk += dKd * fL
    db -= dKd * Kd
    db[L - 1] += np.sum(dKd * Kd, axis=0)
    db[L - 1] += dGL * GL
    dg = np.cumsum(db[::-1], axis=0)[::-1]
    return dq, dk, dv, dg, dbeta, dS


def _chunk_forward_state(S, q, k, v, g, beta):
    """The state after one chunk (the forward of ``chunkwise._chunk``, state only)."""
    L = q.shape[0]
    b = np.cumsum(g, axis=0)
    lower = np.tril(np.ones((L, L)), 0)
    lower_strict = np.tril(np.ones((L, L)), -1)
    diff = b[:, None, :] - b[None, :, :]
    E = np.exp(np.where(lower[:, :, None] > 0, diff, 0.0)) * lower[:, :, None]
    A = beta[:, None] * np.einsum("rc,ic,ric->ri", k, k, E) * lower_strict
    T = unit_lower_inverse(A)
    Ut = T @ (beta[:, None] * v - beta[:, None] * ((k * np.exp(b)) @ S))
    return np.exp(b[L - 1])[:, None] * S + (k * np.exp(b[L - 1][None, :] - b)).T @ Ut


def kda_chunkwise_backward(q, k, v, g, beta, do, s0=None, ds_final=None, scale=1.0, chunk=64):
    """Same conventions and results as ``kda_recurrent_backward``: q, k, v, g, do
    [B,T,H,D] (or [T,H,D]), beta [B,T,H]; returns dq, dk, dv, dg, dbeta, ds0."""
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
    bounds = [(t0, min(t0 + chunk, T)) for t0 in range(0, T, chunk)]
    for bb in range(B):
        for h in range(H):
            sl = lambda x, t0, t1: x[bb, t0:t1, h]  # noqa: E731
            starts = []
            S = S0[bb, h].copy()
            for t0, t1 in bounds:
                starts.append(S)
                S = _chunk_forward_state(S, scale * sl(q, t0, t1), sl(k, t0, t1), sl(v, t0, t1), sl(g, t0, t1),
                                         sl(beta, t0, t1))
            G = G0[bb, h].copy()
            for (t0, t1), S in zip(reversed(bounds), reversed(starts)):
                r = _chunk_backward(S, scale * sl(q, t0, t1), sl(k, t0, t1), sl(v, t0, t1), sl(g, t0, t1),
                                    sl(beta, t0, t1), sl(do, t0, t1), G)
                dq[bb, t0:t1, h] = scale * r[0]
                dk[bb, t0:t1, h] = r[1]
                dv[bb, t0:t1, h] = r[2]
                dg[bb, t0:t1, h] = r[3]
                dbeta[bb, t0:t1, h] = r[4]
                G = r[5]
            ds0[bb, h] = G
    if squeeze:
        dq, dk, dv, dg, dbeta = (x[0] for x in (dq, dk, dv, dg, dbeta))
    return dq, dk, dv, dg, dbeta, ds0
