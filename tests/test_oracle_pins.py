"""Pins for the oracle: facts fixed by the pages and by plain mathematics.

Each test checks the fp64 oracle against something other than itself, chosen
so that a plausible mistake (a dropped term, a wrong sign or index, decay
applied after the write, a transposed state, a wrong cumulative-decay bound)
fails at least one of them.  Equations are from "Kimi Linear: An Expressive,
Efficient Attention Architecture" (research notes), section Method / "From
Linear Attention to KDA" unless stated otherwise.
"""
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_inputs(rng, B=1, T=37, H=2, DK=8, DV=6, gate=0.3, s0=True):
    q = rng.standard_normal((B, T, H, DK))
    k = rng.standard_normal((B, T, H, DK))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, DV))
    g = -gate * np.log1p(np.exp(rng.standard_normal((B, T, H, DK))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    S0 = 0.3 * rng.standard_normal((B, H, DK, DV)) if s0 else None
    return q, k, v, g, beta, S0


def rel(a, b):
    return np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(np.asarray(b)), 1e-300)


# --- 1. one online gradient step on the reconstruction loss (autograd) -------
def test_gradient_step_autograd():
    """DeltaNet is one online GD step on L(S) = 1/2 ||S^T k - v||^2; KDA takes
    that step after the per-channel decay.  The gradient here comes from
    torch.autograd, not from a retyped update formula."""
    rng = np.random.default_rng(0)
    q, k, v, g, beta, S0 = rand_inputs(rng, T=12, H=1)
    o_ref, s_ref = oracle.kda_recurrent(q, k, v, g, beta, s0=S0)
    S = torch.tensor(S0[0, 0])
    outs = []
    for t in range(12):
        St = (torch.exp(torch.tensor(g[0, t, 0]))[:, None] * S).detach().requires_grad_(True)
        kt, vt, qt = (torch.tensor(a[0, t, 0]) for a in (k, v, q))
        loss = 0.5 * ((St.T @ kt - vt) ** 2).sum()
        (grad,) = torch.autograd.grad(loss, St)
        S = (St - float(beta[0, t, 0]) * grad).detach()
        outs.append((S.T @ qt).numpy())
    assert rel(np.stack(outs), o_ref[0, :, 0]) < 1e-13
    assert rel(S.numpy(), s_ref[0, 0]) < 1e-13


def test_deltanet_special_case_autograd():
    """alpha == 1 (g = 0) is DeltaNet: S_t = S_{t-1} - beta grad L(S_{t-1})."""
    rng = np.random.default_rng(1)
    q, k, v, g, beta, S0 = rand_inputs(rng, T=10, H=1)
    g[:] = 0.0
    o_ref, s_ref = oracle.kda_recurrent(q, k, v, g, beta, s0=S0)
    S = torch.tensor(S0[0, 0])
    for t in range(10):
        S = S.detach().requires_grad_(True)
        kt, vt = torch.tensor(k[0, t, 0]), torch.tensor(v[0, t, 0])
        (grad,) = torch.autograd.grad(0.5 * ((S.T @ kt - vt) ** 2).sum(), S)
        S = S - float(beta[0, t, 0]) * grad
    assert rel(S.detach().numpy(), s_ref[0, 0]) < 1e-13


# --- 2. scalar gate: Gated DeltaNet == DeltaNet on rescaled values ------------
def test_gdn_scalar_gate_rescaling_identity():
    """With one decay per head (GDN), Diag(alpha) = alpha I commutes with the
    Householder factor, so with A_t = prod_{s<=t} alpha_s the state is
    S_t = A_t * DeltaNet(v_t / A_t) and o_t = A_t * (DeltaNet state)^T q_t.
    Applying the decay after the write, or per key row with the wrong index,
    breaks this identity."""
    rng = np.random.default_rng(2)
    q, k, v, g, beta, _ = rand_inputs(rng, T=25, H=2, s0=False)
    gs = g[..., :1].repeat(g.shape[-1], axis=-1)          # one value per (t, h)
    o_gdn, s_gdn = oracle.kda_recurrent(q, k, v, gs, beta)
    A = np.exp(np.cumsum(gs[..., 0], axis=1))               # [B,T,H]
    o_dn, s_dn = oracle.kda_recurrent(q, k, v / A[..., None], np.zeros_like(gs), beta)
    assert rel(o_gdn, A[..., None] * o_dn) < 1e-12
    assert rel(s_gdn, A[:, -1][..., None, None] * s_dn) < 1e-12


# --- 3/4. beta = 0: pure decay, closed form ------------------------------------
def test_beta_zero_identity_gate_keeps_state():
    rng = np.random.default_rng(3)
    q, k, v, g, beta, S0 = rand_inputs(rng, T=9)
    o, s = oracle.kda_recurrent(q, k, v, np.zeros_like(g), np.zeros_like(beta), s0=S0)
    assert np.array_equal(s, S0)
    np.testing.assert_allclose(o, np.einsum("bhij,bthi->bthj", S0, q), rtol=0, atol=1e-14)


def test_beta_zero_closed_form_decay():
    """beta = 0: S_t = Diag(exp(sum_{s<=t} g_s)) S_0 exactly."""
    rng = np.random.default_rng(4)
    q, k, v, g, beta, S0 = rand_inputs(rng, T=15)
    o, s = oracle.kda_recurrent(q, k, v, g, np.zeros_like(beta), s0=S0)
    cum = np.exp(np.cumsum(g, axis=1))                      # [B,T,H,DK]
    St = cum[..., :, None] * S0[:, None]                    # [B,T,H,DK,DV]
    np.testing.assert_allclose(s, St[:, -1], rtol=1e-13, atol=0)
    np.testing.assert_allclose(o, np.einsum("bthij,bthi->bthj", St, q), rtol=1e-12, atol=1e-15)


# --- 5. residual form == product form -------------------------------------------
def test_residual_form_equals_product_form():
    rng = np.random.default_rng(5)
    q, k, v, g, beta, S0 = rand_inputs(rng, B=2, T=31, H=3)
    o1, s1 = oracle.kda_recurrent(q, k, v, g, beta, s0=S0, scale=0.7)
    o2, s2 = oracle.kda_recurrent_product(q, k, v, g, beta, s0=S0, scale=0.7)
    assert rel(o1, o2) < 1e-13 and rel(s1, s2) < 1e-13


# --- 6. chunkwise == recurrence ----------------------------------------------------
@pytest.mark.parametrize("chunk", [1, 5, 16, 64])
def test_chunkwise_equals_recurrence(chunk):
    rng = np.random.default_rng(6)
    q, k, v, g, beta, S0 = rand_inputs(rng, B=2, T=150, H=2, DK=16, DV=12)
    o1, s1 = oracle.kda_recurrent(q, k, v, g, beta, s0=S0, scale=0.9)
    o2, s2 = oracle.kda_chunkwise(q, k, v, g, beta, s0=S0, scale=0.9, chunk=chunk)
    assert rel(o2, o1) < 1e-12 and rel(s2, s1) < 1e-12


def test_chunkwise_strong_decay():
    """Gates strong enough that exp(b) spans hundreds of nats inside a chunk."""
    rng = np.random.default_rng(7)
    q, k, v, g, beta, S0 = rand_inputs(rng, T=130, DK=16, DV=8, gate=6.0)
    o1, s1 = oracle.kda_recurrent(q, k, v, g, beta, s0=S0)
    o2, s2 = oracle.kda_chunkwise(q, k, v, g, beta, s0=S0, chunk=64)
    assert rel(o2, o1) < 1e-12 and rel(s2, s1) < 1e-11


def test_unit_lower_inverse():
    rng = np.random.default_rng(8)
    A = np.tril(rng.standard_normal((40, 40)), -1) * 0.3
    T = oracle.chunkwise.unit_lower_inverse(A)
    np.testing.assert_allclose(T @ (np.eye(40) + A), np.eye(40), atol=1e-10)


# --- 7. associative recall / overwrite -----------------------------------------------
def test_recall_of_orthonormal_keys_and_overwrite():
    """alpha == 1, beta == 1, keys = distinct basis vectors: querying e_j returns
    exactly the value written under e_j; writing the same key again keeps only
    the last value (the delta rule overwrites, linear attention would add)."""
    DK = DV = 8
    T = 6
    keys = [0, 3, 5, 3, 7, 1]
    k = np.zeros((1, T, 1, DK))
    for t, i in enumerate(keys):
        k[0, t, 0, i] = 1.0
    rng = np.random.default_rng(9)
    v = rng.standard_normal((1, T, 1, DV))
    q = np.zeros_like(k)
    _, s = oracle.kda_recurrent(q, k, v, np.zeros_like(k), np.ones((1, T, 1)))
    S = s[0, 0]
    for i in range(DK):
        last = [t for t, kk in enumerate(keys) if kk == i]
        want = v[0, last[-1], 0] if last else np.zeros(DV)
        np.testing.assert_allclose(S.T @ np.eye(DK)[i], want, rtol=0, atol=1e-15)


# --- 8. channel wipe ----------------------------------------------------------------
def test_channel_wipe():
    """alpha_c = 0 (g_c = -inf) erases key row c before the write."""
    rng = np.random.default_rng(10)
    q, k, v, g, beta, S0 = rand_inputs(rng, T=1)
    g[:] = 0.0
    g[0, 0, :, 2] = -np.inf
    _, s = oracle.kda_recurrent(q, k, v, g, np.zeros_like(beta), s0=S0)
    assert np.all(s[0, :, 2, :] == 0.0)
    np.testing.assert_array_equal(np.delete(s, 2, axis=2), np.delete(S0, 2, axis=2))


# --- 9. linearity in (V, S0) ---------------------------------------------------------
def test_linearity_in_values_and_initial_state():
    rng = np.random.default_rng(11)
    q, k, v1, g, beta, S1 = rand_inputs(rng, T=20)
    v2 = rng.standard_normal(v1.shape)
    S2 = rng.standard_normal(S1.shape)
    a, b = 0.7, -1.3
    o1, s1 = oracle.kda_recurrent(q, k, v1, g, beta, s0=S1)
    o2, s2 = oracle.kda_recurrent(q, k, v2, g, beta, s0=S2)
    o3, s3 = oracle.kda_recurrent(q, k, a * v1 + b * v2, g, beta, s0=a * S1 + b * S2)
    assert rel(o3, a * o1 + b * o2) < 1e-13 and rel(s3, a * s1 + b * s2) < 1e-13


# --- 10. split invariance / varlen packing ----------------------------------------------
def test_split_invariance():
    rng = np.random.default_rng(12)
    q, k, v, g, beta, S0 = rand_inputs(rng, T=40)
    o, s = oracle.kda_recurrent(q, k, v, g, beta, s0=S0)
    cut = 17
    oa, sa = oracle.kda_recurrent(q[:, :cut], k[:, :cut], v[:, :cut], g[:, :cut], beta[:, :cut], s0=S0)
    ob, sb = oracle.kda_recurrent(q[:, cut:], k[:, cut:], v[:, cut:], g[:, cut:], beta[:, cut:], s0=sa)
    np.testing.assert_array_equal(np.concatenate([oa, ob], axis=1), o)
    np.testing.assert_array_equal(sb, s)


def test_packed_sequences_equal_separate_runs():
    rng = np.random.default_rng(13)
    lens = [5, 64, 1, 70]
    cu = np.concatenate([[0], np.cumsum(lens)])
    Tt = int(cu[-1])
    q, k, v, g, beta, _ = rand_inputs(rng, T=Tt)
    S0 = rng.standard_normal((len(lens), 2, 8, 6))
    o, s = oracle.kda_recurrent(q[0], k[0], v[0], g[0], beta[0], s0=S0, cu=cu)
    oc, sc = oracle.kda_chunkwise(q[0], k[0], v[0], g[0], beta[0], s0=S0, cu=cu, chunk=16)
    for n in range(len(lens)):
        t0, t1 = cu[n], cu[n + 1]
        on, sn = oracle.kda_recurrent(q[:, t0:t1], k[:, t0:t1], v[:, t0:t1], g[:, t0:t1], beta[:, t0:t1],
                                      s0=S0[n:n + 1])
        np.testing.assert_array_equal(o[t0:t1], on[0])
        np.testing.assert_array_equal(s[n], sn[0])
    assert rel(oc, o) < 1e-12 and rel(sc, s) < 1e-12


# --- 11. hand-derived golden example ---------------------------------------------
def test_golden_tiny_example():
    rows, S_want = [], None
    with open(os.path.join(GOLDEN, "kda_tiny_d2.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            parts = line.split()
            if parts[0] == "S":
                S_want = np.array([float(x) for x in parts[1:]]).reshape(2, 2)
            else:
                rows.append([float(x) for x in parts[1:]])
    rows = np.array(rows)
    alpha, beta = rows[:, 0:2], rows[:, 2]
    k, v, q, o_want = rows[:, 3:5], rows[:, 5:7], rows[:, 7:9], rows[:, 9:11]
    f = lambda a: a[None, :, None, :]  # noqa: E731
    o, s = oracle.kda_recurrent(f(q), f(k), f(v), f(np.log(alpha)), beta[None, :, None])
    np.testing.assert_allclose(o[0, :, 0], o_want, atol=1e-14)
    np.testing.assert_allclose(s[0, 0], S_want, atol=1e-14)
    oc, sc = oracle.kda_chunkwise(f(q), f(k), f(v), f(np.log(alpha)), beta[None, :, None], chunk=2)
    np.testing.assert_allclose(oc[0, :, 0], o_want, atol=1e-14)
    np.testing.assert_allclose(sc[0, 0], S_want, atol=1e-14)


# --- generic DPLR ---------------------------------------------------------------------
def test_dplr_without_low_rank_is_gated_linear_attention():
    """a = 0: S_t = Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T has the closed form
    S_T = Diag(G_T) S_0 + sum_t Diag(G_T / G_t) beta_t k_t v_t^T, G_t = exp(sum_{s<=t} g_s)."""
    rng = np.random.default_rng(14)
    q, k, v, g, beta, S0 = rand_inputs(rng, T=12)
    z = np.zeros_like(k)
    _, s = oracle.dplr_recurrent(q, k, v, g, beta, z, z, s0=S0)
    G = np.cumsum(g, axis=1)
    want = np.exp(G[:, -1])[..., None] * S0
    want = want + np.einsum("bthi,bth,bthi,bthj->bhij", np.exp(G[:, -1:] - G), beta, k, v)
    assert rel(s, want) < 1e-13


def test_dplr_tied_keys_is_kda():
    rng = np.random.default_rng(15)
    q, k, v, g, beta, S0 = rand_inputs(rng, T=20)
    o1, s1 = oracle.kda_recurrent(q, k, v, g, beta, s0=S0)
    sb = np.sqrt(beta)[..., None]
    o2, s2 = oracle.dplr_recurrent(q, k, v, g, beta, sb * k, sb * k, s0=S0)
    assert rel(o2, o1) < 1e-13 and rel(s2, s1) < 1e-13


# --- layer pieces against library routines ------------------------------------------
def test_layer_conv_matches_torch_conv1d():
    from oracle import layer as L
    rng = np.random.default_rng(16)
    x = rng.standard_normal((50, 6))
    w = rng.standard_normal((6, 4))
    cu = np.array([0, 20, 21, 50])
    y = L.causal_depthwise_conv(x, w, cu)
    for n in range(3):
        seg = torch.tensor(x[cu[n]:cu[n + 1]]).T[None]
        ref = torch.nn.functional.conv1d(seg, torch.tensor(w)[:, None, :], padding=3, groups=6)[0, :, : seg.shape[-1]]
        np.testing.assert_allclose(y[cu[n]:cu[n + 1]], ref.T.numpy(), atol=1e-13)


def test_layer_norms_and_activations_match_torch():
    from oracle import layer as L
    rng = np.random.default_rng(17)
    x = rng.standard_normal((7, 3 * 16))
    t = torch.tensor(x)
    np.testing.assert_allclose(L.silu(x), torch.nn.functional.silu(t).numpy(), atol=1e-14)
    np.testing.assert_allclose(L.softplus(x), torch.nn.functional.softplus(t).numpy(), atol=1e-14)
    np.testing.assert_allclose(L.sigmoid(x), torch.sigmoid(t).numpy(), atol=1e-14)
    np.testing.assert_allclose(L.l2norm_heads(x, 3).reshape(7, 48),
                               torch.nn.functional.normalize(t.reshape(7, 3, 16), dim=-1, eps=0).reshape(7, 48).numpy(),
                               atol=1e-6)
    w = rng.standard_normal(16)
    np.testing.assert_allclose(L.rmsnorm_heads(x.reshape(7, 3, 16), w),
                               torch.nn.functional.rms_norm(t.reshape(7, 3, 16), (16,), torch.tensor(w), eps=1e-5).numpy(),
                               atol=1e-13)


def test_layer_packed_equals_separate():
    from oracle import layer as L
    import synth
    x, W, cu = synth.layer_inputs(d_model=32, H=2, Ttot=40, nseq=3, rank=8, seed=3)
    W = {n: t.double().numpy() for n, t in W.items()}
    W["W_q"], W["W_k"], W["W_v"] = (np.random.default_rng(0).standard_normal((256, 32)) * 0.1 for _ in range(3))
    x = x.double().numpy()
    y, s = L.kda_layer(x, W, cu, H=2)
    for n in range(3):
        t0, t1 = cu[n], cu[n + 1]
        yn, sn = L.kda_layer(x[t0:t1], W, [0, t1 - t0], H=2)
        np.testing.assert_allclose(y[t0:t1], yn, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(s[n], sn[0], rtol=1e-12, atol=1e-14)


# --- 12. hand-derived golden example of the layer --------------------------------------
def _load_layer_golden():
    """Evaluate tests/golden/kda_layer_tiny.txt line by line (closed forms derived by
    hand; silu and sigmoid are torch's, log and sqrt are math's)."""
    import math

    def _f(fn):
        return lambda u: float(fn(torch.tensor(float(u), dtype=torch.float64)))

    ns = {"log": math.log, "sqrt": math.sqrt, "silu": _f(torch.nn.functional.silu), "sigmoid": _f(torch.sigmoid),
          "vec": lambda *a: np.array(a, dtype=np.float64)}
    with open(os.path.join(GOLDEN, "kda_layer_tiny.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            name, expr = (s.strip() for s in line.split("=", 1))
            ns[name] = eval(expr, {"__builtins__": {}}, ns)  # noqa: S307 (a committed test fixture)
    return ns


_LAYER_WEIGHTS = ("W_q", "W_k", "W_v", "conv_q", "conv_k", "conv_v", "W_adown", "W_aup", "W_gdown", "W_gup",
                  "W_b", "norm_w", "W_o")


def test_layer_golden_tiny_example():
    """The layer's assembly, stage by stage, against a hand-derived example: q, k
    after ShortConv, SiLU and the per-head L2 norm; v; the decay alpha; beta; the
    output gate; then y and the final state through the recurrence, the per-head
    RMSNorm times the gate and the output projection."""
    from oracle import layer as L
    ns = _load_layer_golden()
    W = {n: np.array(ns[n], dtype=np.float64) for n in _LAYER_WEIGHTS}
    x, cu = np.array(ns["x"], dtype=np.float64), ns["cu"]
    q, k, v, g, beta, gate = L.layer_reference_parts(x, W, cu, 2)
    np.testing.assert_allclose(q, np.array(ns["q"]), atol=1e-13)
    np.testing.assert_allclose(k, np.array(ns["k"]), atol=1e-13)
    np.testing.assert_allclose(v, np.array(ns["v"]), atol=1e-13)
    np.testing.assert_allclose(np.exp(g), np.array(ns["alpha"]), atol=1e-13)
    np.testing.assert_allclose(beta, np.array(ns["beta"]), atol=1e-13)
    np.testing.assert_allclose(L.sigmoid(gate), np.array(ns["sg"]), atol=1e-13)
    y, S = oracle.kda_layer(x, W, cu, 2, s0=np.array(ns["S0"], dtype=np.float64))
    np.testing.assert_allclose(S, np.array(ns["S_final"]), atol=1e-13)
    np.testing.assert_allclose(y, np.array(ns["y"]), atol=1e-12)


@pytest.mark.parametrize("swap", [("W_q", "W_k"), ("conv_q", "conv_k")])
def test_layer_golden_detects_swapped_projections(swap):
    """The example is asymmetric: the same oracle fed W_q and W_k (or the q and k
    convolution taps) the other way round misses the hand-derived y."""
    ns = _load_layer_golden()
    W = {n: np.array(ns[n], dtype=np.float64) for n in _LAYER_WEIGHTS}
    W[swap[0]], W[swap[1]] = W[swap[1]], W[swap[0]]
    y, _ = oracle.kda_layer(np.array(ns["x"], dtype=np.float64), W, ns["cu"], 2,
                            s0=np.array(ns["S0"], dtype=np.float64))
    assert np.abs(y - np.array(ns["y"])).max() > 1e-2
