"""kda_gdn_chunk_fwd (one log-gate per token and head) vs the fp64 oracle.

The oracle runs its per-channel recurrence with that gate broadcast over the
128 key channels, which is the gated DeltaNet recurrence by definition (the
per-head scalar forgetting rate of "Kimi Linear", section "From Linear
Attention to KDA"); the broadcast reading itself is pinned on the CPU by the
GDN rescaling identity in test_oracle_pins.py.  Tolerance as for
kda_chunk_fwd: relative L2 <= 1e-2 on o and on the final state."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import f64, rel_l2

pytestmark = pytest.mark.gpu
TOL = 1e-2


def gdn_inputs(**kw):
    inp = synth.op_inputs(scalar_gate=True, **kw)
    inp["gs"] = inp["g"][..., 0].contiguous()  # [B,T,H]: the per-head gate the entry point takes
    return inp


def run_both(kda, inp, scale=1.0, l2=False, heads=None, dtype=None):
    q, k, v, g, gs, beta = (inp[n] for n in ("q", "k", "v", "g", "gs", "beta"))
    if dtype is not None:
        q, k, v = (t.to(dtype) for t in (q, k, v))
    cu = inp.get("cu_seqlens")
    s0 = inp.get("s0")
    o, fs = kda.gdn_chunk_fwd(q.cuda(), k.cuda(), v.cuda(), gs.cuda(), beta.cuda(),
                              initial_state=None if s0 is None else s0.cuda(),
                              cu_seqlens=None if cu is None else cu.cuda(), scale=scale, l2norm_qk=l2)
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    if heads is not None:
        hs = torch.as_tensor(heads).to(q.device)
        q, k, v, g, beta = (t.index_select(2, hs) for t in (q, k, v, g, beta))
        o = o.index_select(2, hs.to(o.device))
        fs = fs.index_select(1, hs.to(fs.device))
        s0 = None if s0 is None else s0.index_select(1, hs.to(s0.device))
    qn, kn = f64(q), f64(k)
    if l2:
        qn = qn / np.sqrt((qn * qn).sum(-1, keepdims=True) + 1e-6)
        kn = kn / np.sqrt((kn * kn).sum(-1, keepdims=True) + 1e-6)
    if cu is None:
        o_ref, s_ref = oracle.kda_recurrent(qn, kn, f64(v), f64(g), f64(beta), s0=f64(s0), scale=scale)
        o_got = f64(o)
    else:
        o_ref, s_ref = oracle.kda_recurrent(qn[0], kn[0], f64(v)[0], f64(g)[0], f64(beta)[0], s0=f64(s0),
                                            cu=cu.cpu().numpy(), scale=scale)
        o_got = f64(o)[0]
    s_got = f64(fs)
    assert np.isfinite(o_got).all() and np.isfinite(s_got).all()
    eo, es = rel_l2(o_got, o_ref), rel_l2(s_got, s_ref)
    print(f"rel-L2 o={eo:.3e} state={es:.3e}")
    return eo, es


@pytest.mark.parametrize("B,T,H", [(1, 64, 1), (1, 1, 2), (2, 63, 2), (1, 65, 3), (2, 200, 3), (3, 130, 5)])
def test_gdn_small_shapes_with_state(kda, B, T, H):
    eo, es = run_both(kda, gdn_inputs(B=B, H=H, T=T, s0_std=0.02, seed=200 + T), scale=0.9)
    assert eo < TOL and es < TOL, (eo, es)


def test_gdn_fp32_inputs_zero_state(kda):
    eo, es = run_both(kda, gdn_inputs(B=1, H=2, T=256, seed=1, dtype=torch.float32))
    assert eo < TOL and es < TOL, (eo, es)


def test_gdn_no_segment_scan_path(kda):
    eo, es = run_both(kda, gdn_inputs(B=4, H=40, T=300, s0_std=0.02, seed=21), heads=[0, 13, 39])
    assert eo < TOL and es < TOL, (eo, es)


def test_gdn_strong_decay_exact_fallback(kda):
    """Per-head gates ~30x stronger: the chunk's decay range exceeds the
    factored path's bound and chunks take the exact fallback."""
    eo, es = run_both(kda, gdn_inputs(B=1, H=2, T=257, gate_scale=3.0, s0_std=0.02, seed=22))
    assert eo < TOL and es < TOL, (eo, es)


def test_gdn_mixed_decay_and_l2norm(kda):
    inp = gdn_inputs(B=1, H=2, T=512, gate_scale=1.0, s0_std=0.02, seed=23)
    inp["gs"][:, 200:300] *= 4.0
    inp["g"][:, 200:300] *= 4.0
    inp["q"] = (inp["q"].float() * 3.0).bfloat16()
    eo, es = run_both(kda, inp, l2=True)
    assert eo < TOL and es < TOL, (eo, es)


def test_gdn_varlen_with_empty_sequences(kda):
    cu = [0, 0, 5, 69, 70, 70, 300, 301, 600]
    eo, es = run_both(kda, gdn_inputs(B=len(cu) - 1, H=3, T=cu[-1], s0_std=0.02, seed=24, cu_seqlens=cu))
    assert eo < TOL and es < TOL, (eo, es)


def test_gdn_matches_per_channel_entry_point(kda):
    """The same problem through kda_chunk_fwd with the gate broadcast over channels."""
    inp = gdn_inputs(B=1, H=4, T=1000, s0_std=0.02, seed=25)
    args = [inp[n].cuda() for n in ("q", "k", "v")]
    o1, s1 = kda.gdn_chunk_fwd(*args, inp["gs"].cuda(), inp["beta"].cuda(), initial_state=inp["s0"].cuda())
    o2, s2 = kda.chunk_fwd(*args, inp["g"].cuda(), inp["beta"].cuda(), initial_state=inp["s0"].cuda())
    torch.cuda.synchronize()
    d_o, d_s = rel_l2(f64(o1), f64(o2)), rel_l2(f64(s1), f64(s2))
    print(f"gdn vs per-channel: o {d_o:.2e} state {d_s:.2e}")
    assert d_o < 5e-3 and d_s < 5e-3


def test_gdn_deterministic_bits(kda):
    inp = gdn_inputs(B=1, H=2, T=700, s0_std=0.02, seed=26)
    a = [kda.gdn_chunk_fwd(*(inp[n].cuda() for n in ("q", "k", "v", "gs", "beta")), initial_state=inp["s0"].cuda())
         for _ in range(2)]
    assert torch.equal(a[0][0], a[1][0]) and torch.equal(a[0][1], a[1][1])


def test_gdn_prefill_4k_full(kda):
    eo, es = run_both(kda, gdn_inputs(**{**synth.PREFILL_4K, "seed": 27}))
    assert eo < TOL and es < TOL, (eo, es)


@pytest.mark.slow
def test_gdn_prefill_64k_sampled_heads(kda):
    """B=1, H=16, T=65536 in the bench's launch configuration; heads 3, 7, 12 and 14."""
    inp = gdn_inputs(**{**synth.prefill_sweep(65536), "device": "cuda"})
    eo, es = run_both(kda, inp, heads=[3, 7, 12, 14])
    assert eo < TOL and es < TOL, (eo, es)


def test_balanced_plan_packed_sequences(kda):
    """Packed sequences with 128 (sequence, head) pairs take the device-made
    balanced plan; the scalar-gate kernels share it."""
    cu = [0, 100, 5100, 5164, 7164, 7165, 11165, 11900, 12000]
    assert kda.chunk_fwd_segments(1, cu[-1], 16, len(cu) - 1) == (-1, -1)
    inp = gdn_inputs(B=len(cu) - 1, H=16, T=cu[-1], s0_std=0.02, seed=33, cu_seqlens=cu)
    eo, es = run_both(kda, inp, heads=[1, 14])
    assert eo < TOL and es < TOL, (eo, es)
