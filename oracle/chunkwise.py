"""Naive chunkwise KDA -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.

A plain fp64 numpy statement of the chunkwise form of KDA, one chunk at a
time, no blocking or fusion beyond the chunk itself.

Source: "Kimi Linear: An Expressive, Efficient Attention Architecture"
(research notes), section "Chunkwise Algorithm" (split into chunks of C = 64;
unroll the per-channel decay and rank-1 corrections inside a chunk; pack them
with the WY representation; invert the triangular system with the UT
transform; only the fixed-size state crosses chunks), with the cumulative
decay as corrected in section "Mathematical Rigor":
gamma^{i->j} = prod_{k=i+1}^{j} alpha^k and gamma^r = prod_{k=1}^{r} alpha^k.
The news rewrite of the report ("Kimi Linear", m.jxzklqfsx.com) adds that the
lower-triangular inverse is taken by forward substitution, row by row, and
that the output is the inter-chunk recurrence plus an intra-chunk parallel
term.  Its displayed formulas were lost in extraction, so the chunk equations
below are the plainest reading that reproduces the recurrence.  Derivation:
with u~_i = beta_i (v_i - S~_{i-1}^T k_i) the recurrence unrolls inside a chunk
to S_r = Diag(gamma_r) S + sum_{i<=r} Diag(gamma_r / gamma_i) k_i u~_i^T.
Substituting S~_{r-1} = Diag(alpha_r) S_{r-1} into u~_r gives
u~_r + sum_{i<r} A[r,i] u~_i = beta_r v_r - beta_r (gamma_r (.) k_r)^T S, i.e.
(I + A) U~ = diag(beta) V - diag(beta) (K (.) gamma) S; reading o_r = S_r^T q_r
and S_{L-1} off the same unrolled sum gives O and S_next.  The tests pin the
result against the token-by-token recurrence for several chunk sizes.

Per chunk with rows r = 0..L-1 (L <= C) and entering state S (DK x DV):

  b_r      = sum_{s <= r} g_s                    (log-space cumulative decay)
  gamma_r  = exp(b_r)
  A[r,i]   = beta_r * sum_c k[r,c] k[i,c] exp(b[r,c] - b[i,c])   (i < r)
  P[r,i]   =          sum_c q[r,c] k[i,c] exp(b[r,c] - b[i,c])   (i <= r)
  U~       = (I + A)^{-1} (diag(beta) V - diag(beta) (K (.) gamma) S)
  O        = (Q (.) gamma) S + P U~
  S_next   = Diag(gamma_{L-1}) S + (K (.) exp(b_{L-1} - b))^T U~
"""
from __future__ import annotations

import numpy as np


def unit_lower_inverse(A: np.ndarray) -> np.ndarray:
    """(I + A)^{-1} for strictly lower-triangular A, by forward substitution.

    Row r of T = (I + A)^{-1} solves T[r] = e_r - sum_{j<r} A[r, j] T[j]
    (from (I + A) T = I read row by row), taken in increasing r.
    """
    n = A.shape[0]
    T = np.zeros_like(A)
    for r in range(n):
        row = np.zeros(n)
        row[r] = 1.0
        for j in range(r):
            if A[r, j] != 0.0:
                row -= A[r, j] * T[j]
        T[r] = row
    return T


def _chunk(S, q, k, v, g, beta):
    L = q.shape[0]
    b = np.cumsum(g, axis=0)                              # [L, DK]
    gamma = np.exp(b)
    diff = b[:, None, :] - b[None, :, :]                  # [r, i, c] = b_r - b_i
    lower_strict = np.tril(np.ones((L, L)), -1)
    lower = np.tril(np.ones((L, L)), 0)
    # exp() only where i <= r, where the exponent is <= 0 for g <= 0
    ex = np.exp(np.where(lower[:, :, None] > 0, diff, 0.0))
    A = beta[:, None] * np.einsum("rc,ic,ric->ri", k, k, ex) * lower_strict
    P = np.einsum("rc,ic,ric->ri", q, k, ex) * lower
    T = unit_lower_inverse(A)
    rhs = beta[:, None] * v - beta[:, None] * ((k * gamma) @ S)
    U = T @ rhs
    O = (q * gamma) @ S + P @ U
    S_next = gamma[L - 1][:, None] * S + (k * np.exp(b[L - 1][None, :] - b)).T @ U
    return O, S_next


def kda_chunkwise(q, k, v, g, beta, s0=None, cu=None, scale=1.0, chunk=64):
    """Chunkwise KDA in fp64.  Same conventions as ``oracle.kda_recurrent``."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    dense = cu is None
    if dense:
        B, T, H, DK = q.shape
        DV = v.shape[-1]
        cu = np.arange(B + 1) * T
        q, k, g = (a.reshape(B * T, H, DK) for a in (q, k, g))
        v = v.reshape(B * T, H, DV)
        beta = beta.reshape(B * T, H)
    cu = np.asarray(cu, dtype=np.int64)
    N = len(cu) - 1
    H, DK, DV = q.shape[1], q.shape[2], v.shape[2]
    o = np.zeros((q.shape[0], H, DV))
    sT = np.zeros((N, H, DK, DV))
    for n in range(N):
        for h in range(H):
            S = np.zeros((DK, DV)) if s0 is None else np.array(np.asarray(s0, dtype=np.float64).reshape(N, H, DK, DV)[n, h])
            for t0 in range(int(cu[n]), int(cu[n + 1]), chunk):
                t1 = min(t0 + chunk, int(cu[n + 1]))
                O, S = _chunk(S, scale * q[t0:t1, h], k[t0:t1, h], v[t0:t1, h], g[t0:t1, h], beta[t0:t1, h])
                o[t0:t1, h] = O
            sT[n, h] = S
    if dense:
        o = o.reshape(B, T, H, DV)
    return o, sT
