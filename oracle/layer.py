"""KDA layer forward -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.

Plain fp64 numpy statement of the KDA layer around the operator.

Source: "Kimi Linear: An Expressive, Efficient Attention Architecture"
(research notes), section "Neural Parameterization" (table: bias-free Q/K/V
projections; depthwise ShortConv, kernel 4; SiLU after the Q/K/V convolutions;
L2 normalisation of q and k; per-channel alpha from a low-rank down/up
projection of rank 128; a sigmoid scalar beta per token and head; RMSNorm and
a low-rank sigmoid output gate) and section "Code Verification" (three
kernel-size-4 ShortConvolutions; b_proj(...).sigmoid(); hidden -> 128 -> 4096
alpha gate; FusedRMSNormGated with activation 'sigmoid').  The news rewrite
("Kimi Linear", m.jxzklqfsx.com, section "Neural parameterization") adds that
the per-head RMSNorm and the data-dependent gate come before the output
projection.  Where the pages' formulas were lost (the decay function and the
gate form), the readings are: alpha = exp(-softplus(a)), no extra bias or
A_log; gate = sigmoid(W_up W_down x); RMSNorm eps 1e-5 with a per-channel
weight shared by all heads; L2 norm x / sqrt(sum x^2 + 1e-6); the causal
convolution restarts from zero history at every packed-sequence start.

Weights (row-major, as ``y = x @ W.T``):
  W_q, W_k, W_v [H*D, d_model]; W_adown, W_gdown [rank, d_model];
  W_b [H, d_model]; W_aup [H*D, rank]; W_gup [H*D, rank];
  conv_q, conv_k, conv_v [H*D, 4] (tap j multiplies x[t - 3 + j]);
  norm_w [D]; W_o [d_model, H*D].
"""
from __future__ import annotations

import numpy as np


def silu(x):
    return x / (1.0 + np.exp(-x))


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def softplus(x):
    # log(1 + e^x), written to stay finite for large |x|
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def causal_depthwise_conv(x, w, cu):
    """y[t, ch] = sum_j w[ch, j] * x[t - 3 + j, ch], with x taken as zero before
    the start of the packed sequence that t belongs to."""
    T, C = x.shape
    K = w.shape[1]
    y = np.zeros_like(x)
    for n in range(len(cu) - 1):
        t0, t1 = int(cu[n]), int(cu[n + 1])
        seg = x[t0:t1]
        pad = np.vstack([np.zeros((K - 1, C)), seg])
        for j in range(K):
            y[t0:t1] += w[:, j][None, :] * pad[j:j + (t1 - t0)]
    return y


def l2norm_heads(x, H, eps=1e-6):
    T = x.shape[0]
    xr = x.reshape(T, H, -1)
    return xr / np.sqrt((xr * xr).sum(-1, keepdims=True) + eps)


def rmsnorm_heads(x, w, eps=1e-5):
    return x / np.sqrt((x * x).mean(-1, keepdims=True) + eps) * w


def layer_reference_parts(x, W, cu, H):
    """The layer up to (and excluding) the KDA core: returns q, k, v [T,H,D],
    g [T,H,D] (log decay), beta [T,H] and the output-gate pre-activation."""
    x = np.asarray(x, dtype=np.float64)
    f = lambda name: np.asarray(W[name], dtype=np.float64)  # noqa: E731
    T = x.shape[0]
    q = silu(causal_depthwise_conv(x @ f("W_q").T, f("conv_q"), cu))
    k = silu(causal_depthwise_conv(x @ f("W_k").T, f("conv_k"), cu))
    v = silu(causal_depthwise_conv(x @ f("W_v").T, f("conv_v"), cu))
    q = l2norm_heads(q, H)
    k = l2norm_heads(k, H)
    v = v.reshape(T, H, -1)
    a = (x @ f("W_adown").T) @ f("W_aup").T
    g = -softplus(a).reshape(T, H, -1)
    beta = sigmoid(x @ f("W_b").T)
    gate = ((x @ f("W_gdown").T) @ f("W_gup").T).reshape(T, H, -1)
    return q, k, v, g, beta, gate


def kda_layer(x, W, cu, H, s0=None, core=None):
    """Full layer: returns (y [T, d_model], final state [N,H,D,D]).

    ``core`` is the KDA operator used in the middle (defaults to the
    token-by-token oracle recurrence)."""
    if core is None:
        from . import kda_recurrent as core
    q, k, v, g, beta, gate = layer_reference_parts(x, W, cu, H)
    o, sT = core(q, k, v, g, beta, s0=s0, cu=cu)
    on = rmsnorm_heads(o, np.asarray(W["norm_w"], dtype=np.float64)) * sigmoid(gate)
    y = on.reshape(on.shape[0], -1) @ np.asarray(W["W_o"], dtype=np.float64).T
    return y, sT
