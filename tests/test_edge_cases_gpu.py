"""The method's degenerate cases on the GPU, element by element against the
oracle (relative L2 <= 1e-2 on o and on the final state, the prefill bar).

The cases are those the oracle is pinned on (the CPU pins in
test_oracle_pins.py), now run through the CUDA kernels, where each takes a
different path or boundary:
  * a channel wipe, g = -inf on one key channel ("From Linear Attention to
    KDA": alpha in [0, 1]; alpha = 0 forgets that channel's row of the state):
    the kernel clamps log-gates below -1e4, and the chunk's decay range sends
    it down the exact fallback;
  * beta = 0 with random gates: no writes, the state only decays, and
    o_t = (Diag(gamma_t) S_0)^T q_t;
  * alpha = 1 and beta = 1 on standard-basis keys (DeltaNet, the same
    section): recall of the value last written under the queried key, and
    overwrite when a key is written again;
  * per-channel decay ranges just inside (60 nats) and just outside (70 nats)
    the factored path's bound of 64 nats per chunk, where the gated operands
    reach e^{+-30} and where the exact fallback takes over ("Mathematical
    Rigor": gamma^{i->j} = prod_{k=i+1}^{j} alpha^k)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import f64, rel_l2

pytestmark = pytest.mark.gpu
TOL = 1e-2


def run_both(kda, inp, gdn=False):
    q, k, v, g, beta, s0 = (inp[n] for n in ("q", "k", "v", "g", "beta", "s0"))
    gk = g[..., 0].contiguous() if gdn else g
    fn = kda.gdn_chunk_fwd if gdn else kda.chunk_fwd
    o, fs = fn(q.cuda(), k.cuda(), v.cuda(), gk.cuda(), beta.cuda(), initial_state=None if s0 is None else s0.cuda())
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    o_ref, s_ref = oracle.kda_recurrent(f64(q), f64(k), f64(v), f64(g), f64(beta), s0=f64(s0))
    o_got, s_got = f64(o), f64(fs)
    assert np.isfinite(o_got).all() and np.isfinite(s_got).all()
    eo, es = rel_l2(o_got, o_ref), rel_l2(s_got, s_ref)
    print(f"rel-L2 o={eo:.3e} state={es:.3e}")
    return eo, es, o_got, s_got, o_ref, s_ref


@pytest.mark.parametrize("T,H", [(300, 2), (3000, 16)])
def test_channel_wipe_minus_inf_gate(kda, T, H):
    inp = synth.op_inputs(B=1, H=H, T=T, s0_std=0.02, seed=501)
    inp["g"][0, 70, :, 5] = float("-inf")     # one token wipes channel 5 of every head
    inp["g"][0, T - 10:, 0, 77] = float("-inf")  # the last ten tokens keep wiping channel 77 of head 0
    eo, es, _, s_got, _, s_ref = run_both(kda, inp)
    assert eo < TOL and es < TOL, (eo, es)
    # the last token wiped row 77 of head 0 before its write: only beta_T k_T u_T^T remains there
    assert np.abs(s_got[0, 0, 77] - s_ref[0, 0, 77]).max() < 2e-2 * max(np.abs(s_ref[0, 0, 77]).max(), 1e-3)


@pytest.mark.parametrize("T,H,gate_scale", [(200, 2, 0.1), (3000, 16, 0.01)])
def test_beta_zero_only_decays(kda, T, H, gate_scale):
    # the long case uses weaker gates so that the decayed state stays well inside fp32's range
    inp = synth.op_inputs(B=1, H=H, T=T, gate_scale=gate_scale, s0_std=0.02, seed=502)
    inp["beta"].zero_()
    eo, es, _, s_got, _, s_ref = run_both(kda, inp)
    assert eo < TOL and es < TOL, (eo, es)
    # closed form of the state: S_T = Diag(exp(sum_t g_t)) S_0
    s_closed = np.exp(f64(inp["g"])[0].sum(0))[:, :, None] * f64(inp["s0"])[0]
    assert rel_l2(s_got[0], s_closed) < TOL


def _basis_recall_inputs(T, H, seed):
    inp = synth.op_inputs(B=1, H=H, T=T, s0_std=None, seed=seed)
    idx = (torch.arange(T) * 37) % 128  # 128 distinct keys per 128 tokens, then written again
    key = torch.nn.functional.one_hot(idx, 128).float()
    qidx = (torch.arange(T) * 37 - 37 * 5) % 128  # the key written five tokens earlier
    qry = torch.nn.functional.one_hot(qidx, 128).float()
    inp["k"] = key[None, :, None, :].expand(1, T, H, 128).contiguous().bfloat16()
    inp["q"] = qry[None, :, None, :].expand(1, T, H, 128).contiguous().bfloat16()
    inp["g"].zero_()
    inp["beta"].fill_(1.0)
    return inp


@pytest.mark.parametrize("gdn", [False, True])
def test_deltanet_recall_and_overwrite_on_basis_keys(kda, gdn):
    T, H = 640, 2
    inp = _basis_recall_inputs(T, H, 503)
    eo, es, o_got, _, o_ref, _ = run_both(kda, inp, gdn=gdn)
    assert eo < TOL and es < TOL, (eo, es)
    v = f64(inp["v"])[0]
    # from token 5 on, q_t asks for the key written at t-5, which still holds v_{t-5} exactly
    np.testing.assert_allclose(o_ref[0, 5:], v[:-5], atol=1e-12)
    assert rel_l2(o_got[0, 5:], v[:-5]) < TOL


@pytest.mark.parametrize("nats", [60.0, 70.0])
def test_decay_range_around_the_factored_bound(kda, nats):
    """Channels 0..15 decay by `nats` over the 63 in-chunk steps (g = -nats/63 per
    token); the other channels keep the prefill gates."""
    T, H = 1024, 4
    inp = synth.op_inputs(B=1, H=H, T=T, s0_std=0.02, seed=504 + int(nats))
    inp["g"][..., :16] = -nats / 63.0
    eo, es, *_ = run_both(kda, inp)
    assert eo < TOL and es < TOL, (eo, es)


@pytest.mark.parametrize("nats", [60.0, 70.0])
def test_gdn_decay_range_around_the_factored_bound(kda, nats):
    T, H = 1024, 4
    inp = synth.op_inputs(B=1, H=H, T=T, s0_std=0.02, seed=506 + int(nats), scalar_gate=True)
    inp["g"][:] = -nats / 63.0
    eo, es, *_ = run_both(kda, inp, gdn=True)
    assert eo < TOL and es < TOL, (eo, es)
