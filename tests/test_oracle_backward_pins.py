"""Pins of the oracle's reverse mode (CPU only).

oracle.kda_recurrent_backward is checked against (1) torch autograd on a
separately written torch statement of the forward recurrence (decay, residual
write, o = S^T q), and (2) central finite differences of the C oracle's
forward on tiny inputs.  A dropped term, a wrong sign or a transposed operand in
any reverse line changes one of the six gradients and fails both."""
import numpy as np
import torch

import oracle


def torch_forward(q, k, v, g, beta, s0, scale):
    """[T, D] tensors of one (sequence, head); returns (o [T, D], S_T)."""
    S = s0
    outs = []
    for t in range(q.shape[0]):
        S = torch.exp(g[t])[:, None] * S
        u = beta[t] * (v[t] - S.T @ k[t])
        S = S + torch.outer(k[t], u)
        outs.append(S.T @ (scale * q[t]))
    return torch.stack(outs), S


def rand_problem(T, D, seed, gate=0.3):
    r = np.random.default_rng(seed)
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)  # noqa: E731
    return dict(q=unit(r.standard_normal((T, D))), k=unit(r.standard_normal((T, D))), v=r.standard_normal((T, D)),
                g=-gate * np.log1p(np.exp(r.standard_normal((T, D)))), beta=1 / (1 + np.exp(-r.standard_normal(T))),
                s0=0.3 * r.standard_normal((D, D)), do=r.standard_normal((T, D)), dsT=r.standard_normal((D, D)))


def test_backward_matches_autograd():
    for T, D, scale, seed in ((7, 5, 1.0, 1), (40, 8, 0.7, 2), (3, 2, 1.3, 3)):
        p = rand_problem(T, D, seed)
        tt = {n: torch.tensor(p[n], dtype=torch.float64, requires_grad=n not in ("do", "dsT")) for n in p}
        o, ST = torch_forward(tt["q"], tt["k"], tt["v"], tt["g"], tt["beta"], tt["s0"], scale)
        loss = (o * tt["do"]).sum() + (ST * tt["dsT"]).sum()
        loss.backward()
        sh = lambda x: x[:, None, :]  # noqa: E731  [T,1,D]: one head
        dq, dk, dv, dg, db, ds0 = oracle.kda_recurrent_backward(
            sh(p["q"]), sh(p["k"]), sh(p["v"]), sh(p["g"]), p["beta"][:, None], sh(p["do"]),
            s0=p["s0"][None, None], ds_final=p["dsT"][None, None], scale=scale)
        for name, got in (("q", dq[:, 0]), ("k", dk[:, 0]), ("v", dv[:, 0]), ("g", dg[:, 0]), ("beta", db[:, 0]),
                          ("s0", ds0[0, 0])):
            ref = tt[name].grad.numpy()
            assert np.allclose(got, ref, rtol=1e-10, atol=1e-12), (name, np.abs(got - ref).max())


def test_backward_matches_finite_differences():
    T, D, scale = 4, 3, 0.9
    p = rand_problem(T, D, 7)

    def loss(pp):
        e = lambda x: x[None, :, None]  # noqa: E731  [1,T,1,...]
        o, sT = oracle.kda_recurrent(e(pp["q"]), e(pp["k"]), e(pp["v"]), e(pp["g"]), e(pp["beta"]),
                                     s0=pp["s0"][None, None], scale=scale)
        return float((o[0, :, 0] * p["do"]).sum() + (sT[0, 0] * p["dsT"]).sum())

    grads = oracle.kda_recurrent_backward(p["q"][:, None], p["k"][:, None], p["v"][:, None], p["g"][:, None],
                                          p["beta"][:, None], p["do"][:, None], s0=p["s0"][None, None],
                                          ds_final=p["dsT"][None, None], scale=scale)
    got = dict(q=grads[0][:, 0], k=grads[1][:, 0], v=grads[2][:, 0], g=grads[3][:, 0], beta=grads[4][:, 0],
               s0=grads[5][0, 0])
    eps = 1e-6
    for name in ("q", "k", "v", "g", "beta", "s0"):
        fd = np.zeros_like(p[name])
        for idx in np.ndindex(p[name].shape):
            hi = {n: x.copy() for n, x in p.items()}
            lo = {n: x.copy() for n, x in p.items()}
            hi[name][idx] += eps
            lo[name][idx] -= eps
            fd[idx] = (loss(hi) - loss(lo)) / (2 * eps)
        assert np.allclose(got[name], fd, rtol=1e-6, atol=1e-8), (name, np.abs(got[name] - fd).max())


def test_backward_batched_heads_match_single():
    """Batch and head dimensions are independent problems."""
    r = np.random.default_rng(11)
    B, T, H, D = 2, 9, 3, 4
    q, k, v, do = (r.standard_normal((B, T, H, D)) for _ in range(4))
    g = -0.2 * np.abs(r.standard_normal((B, T, H, D)))
    beta = r.uniform(0.1, 0.9, (B, T, H))
    s0, dsT = r.standard_normal((B, H, D, D)), r.standard_normal((B, H, D, D))
    full = oracle.kda_recurrent_backward(q, k, v, g, beta, do, s0=s0, ds_final=dsT)
    for b in range(B):
        for h in range(H):
            one = oracle.kda_recurrent_backward(q[b, :, h:h + 1], k[b, :, h:h + 1], v[b, :, h:h + 1],
                                                g[b, :, h:h + 1], beta[b, :, h:h + 1], do[b, :, h:h + 1],
                                                s0=s0[b, h], ds_final=dsT[b, h])
            assert np.allclose(full[0][b, :, h], one[0][:, 0]) and np.allclose(full[3][b, :, h], one[3][:, 0])
            assert np.allclose(full[4][b, :, h], one[4][:, 0]) and np.allclose(full[5][b, h], one[5][0, 0])


def test_chunkwise_backward_equals_recurrent_backward():
    """The chunk-form reverse mode (written from the chunkwise forward, line by line)
    against the token-by-token reverse mode pinned above: chunk sizes from 1 to 64,
    ragged last chunks, strong decay, a q scale, several sequences and heads."""
    cases = ((1, 7, 1, 5, 3, 0.3, 1.0), (2, 40, 2, 6, 16, 0.3, 0.7), (1, 33, 1, 4, 64, 2.0, 1.0),
             (1, 10, 1, 3, 1, 0.3, 1.3), (1, 70, 1, 8, 64, 0.3, 1.0))
    for B, T, H, D, C, gate, scale in cases:
        r = np.random.default_rng(B * 1000 + T)
        unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)  # noqa: E731
        q, k = unit(r.standard_normal((B, T, H, D))), unit(r.standard_normal((B, T, H, D)))
        v = r.standard_normal((B, T, H, D))
        g = -gate * np.log1p(np.exp(r.standard_normal((B, T, H, D))))
        beta = 1 / (1 + np.exp(-r.standard_normal((B, T, H))))
        s0, do, ds = 0.3 * r.standard_normal((B, H, D, D)), r.standard_normal((B, T, H, D)), r.standard_normal((B, H, D, D))
        a = oracle.kda_chunkwise_backward(q, k, v, g, beta, do, s0=s0, ds_final=ds, scale=scale, chunk=C)
        b = oracle.kda_recurrent_backward(q, k, v, g, beta, do, s0=s0, ds_final=ds, scale=scale)
        for name, x, y in zip(("dq", "dk", "dv", "dg", "dbeta", "ds0"), a, b):
            err = np.max(np.abs(x - y)) / np.max(np.abs(y))
            assert err < 1e-12, (B, T, H, D, C, name, err)

