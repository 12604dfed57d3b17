"""kda_dplr_chunk_fwd (the untied DPLR comparison kernel) vs the fp64 oracle.

The oracle runs the product-form recurrence S = (I - a b^T) Diag(exp g) S +
beta k v^T token by token on the same (bf16-rounded) inputs.  Tolerance as for
kda_chunk_fwd: relative L2 <= 1e-2 on o and on the final state."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import f64, rel_l2

pytestmark = pytest.mark.gpu
TOL = 1e-2
NAMES = ("q", "k", "v", "a", "b", "g", "beta")


def run_both(kda, inp, scale=1.0):
    cu = inp.get("cu_seqlens")
    s0 = inp.get("s0")
    o, fs = kda.dplr_chunk_fwd(*(inp[n].cuda() for n in NAMES), initial_state=None if s0 is None else s0.cuda(),
                               cu_seqlens=None if cu is None else cu.cuda(), scale=scale)
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    args = [f64(inp[n]) for n in ("q", "k", "v", "g", "beta", "a", "b")]
    if cu is None:
        o_ref, s_ref = oracle.dplr_recurrent(*args, s0=f64(s0), scale=scale)
        o_got = f64(o)
    else:
        o_ref, s_ref = oracle.dplr_recurrent(*(x[0] for x in args), s0=f64(s0), cu=cu.cpu().numpy(), scale=scale)
        o_got = f64(o)[0]
    s_got = f64(fs)
    assert np.isfinite(o_got).all() and np.isfinite(s_got).all()
    eo, es = rel_l2(o_got, o_ref), rel_l2(s_got, s_ref)
    print(f"rel-L2 o={eo:.3e} state={es:.3e}")
    return eo, es


@pytest.mark.parametrize("B,T,H", [(1, 64, 1), (1, 1, 2), (2, 63, 2), (1, 65, 3), (2, 200, 3), (3, 130, 5)])
def test_dplr_small_shapes_with_state(kda, B, T, H):
    eo, es = run_both(kda, synth.dplr_inputs(B=B, H=H, T=T, s0_std=0.02, seed=400 + T), scale=0.9)
    assert eo < TOL and es < TOL, (eo, es)


def test_dplr_fp32_inputs(kda):
    eo, es = run_both(kda, synth.dplr_inputs(B=1, H=2, T=256, dtype=torch.float32, seed=401))
    assert eo < TOL and es < TOL, (eo, es)


def test_dplr_strong_decay_exact_fallback(kda):
    eo, es = run_both(kda, synth.dplr_inputs(B=1, H=2, T=257, gate_scale=3.0, s0_std=0.02, seed=402))
    assert eo < TOL and es < TOL, (eo, es)


def test_dplr_mixed_decay(kda):
    inp = synth.dplr_inputs(B=1, H=2, T=512, gate_scale=1.0, s0_std=0.02, seed=403)
    inp["g"][:, 200:300] *= 4.0
    eo, es = run_both(kda, inp)
    assert eo < TOL and es < TOL, (eo, es)


def test_dplr_varlen_with_empty_sequences(kda):
    cu = [0, 0, 5, 69, 70, 70, 300, 301, 600]
    eo, es = run_both(kda, synth.dplr_inputs(B=len(cu) - 1, H=3, T=cu[-1], s0_std=0.02, seed=404, cu_seqlens=cu))
    assert eo < TOL and es < TOL, (eo, es)


def test_dplr_tied_case_matches_kda_kernel(kda):
    """a = beta k, b = k is KDA: the DPLR kernel agrees with kda_chunk_fwd."""
    inp = synth.op_inputs(B=1, H=4, T=700, s0_std=0.02, seed=405)
    d = {n: inp[n].cuda() for n in ("q", "k", "v", "g", "beta")}
    a = (d["beta"][..., None] * d["k"].float()).to(d["k"].dtype)
    o1, s1 = kda.dplr_chunk_fwd(d["q"], d["k"], d["v"], a, d["k"], d["g"], d["beta"],
                                initial_state=inp["s0"].cuda())
    o2, s2 = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=inp["s0"].cuda())
    torch.cuda.synchronize()
    d_o, d_s = rel_l2(f64(o1), f64(o2)), rel_l2(f64(s1), f64(s2))
    print(f"tied DPLR vs KDA kernel: o {d_o:.2e} state {d_s:.2e}")
    assert d_o < 1e-2 and d_s < 1e-2


def test_dplr_prefill_4k_full(kda):
    eo, es = run_both(kda, synth.dplr_inputs(B=1, H=16, T=4096, s0_std=0.02, seed=406))
    assert eo < TOL and es < TOL, (eo, es)
