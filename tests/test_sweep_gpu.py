"""The prefill length sweep on the GPU: B=1, H=16, d=128, T in {8K, 16K, 32K,
64K} with the prefill distributions (bf16 q/k/v, fp32 g and beta, random
initial state), for the three prefill kernels the pages compare: KDA
(per-channel gate), gated DeltaNet (the gate broadcast to a per-head scalar)
and the untied DPLR recurrence ("Kimi Linear: An Expressive, Efficient
Attention Architecture", section "Chunkwise Algorithm": kernel time against
length, B=1, 16 heads, up to 64K).

Every length runs in the launch configuration the bench would time (the
segment plan cuts each length differently: ``kda_chunk_fwd_segment_tokens``).
The oracle checks three sampled heads end to end (one for the untied DPLR
kernel, whose product-form oracle costs O(d^3) per token): relative L2 <= 1e-2
on o and on the final state, as for every prefill test."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import f64, rel_l2

pytestmark = pytest.mark.gpu
TOL = 1e-2
HEADS = [1, 8, 14]


def _sub(t, hs, dim):
    return t.index_select(dim, hs.to(t.device))


def _check(o, fs, inp, hs, ref_fn):
    o, fs = _sub(o, hs, 2), _sub(fs, hs, 1)
    args = {n: _sub(inp[n], hs, 2) for n in inp if n not in ("s0", "cu_seqlens")}
    s0 = _sub(inp["s0"], hs, 1)
    o_ref, s_ref = ref_fn({n: f64(t) for n, t in args.items()}, f64(s0))
    o_got, s_got = f64(o), f64(fs)
    assert np.isfinite(o_got).all() and np.isfinite(s_got).all()
    eo, es = rel_l2(o_got, o_ref), rel_l2(s_got, s_ref)
    print(f"rel-L2 o={eo:.3e} state={es:.3e}")
    return eo, es


def _kda_ref(a, s0):
    return oracle.kda_recurrent(a["q"], a["k"], a["v"], a["g"], a["beta"], s0=s0)


@pytest.mark.slow
@pytest.mark.parametrize("T", synth.PREFILL_SWEEP_T[:-1])
def test_kda_sweep_sampled_heads(kda, T):
    inp = synth.op_inputs(**synth.prefill_sweep(T), device="cuda")
    first, mid = kda.chunk_fwd_segments(1, T, 16)
    print(f"T={T}: segments of {first}/{mid} tokens")
    o, fs = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], initial_state=inp["s0"])
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    eo, es = _check(o, fs, inp, torch.tensor(HEADS), _kda_ref)
    assert eo < TOL and es < TOL, (eo, es)


@pytest.mark.slow
@pytest.mark.parametrize("T", synth.PREFILL_SWEEP_T[:-1])
def test_gdn_sweep_sampled_heads(kda, T):
    inp = synth.op_inputs(**{**synth.prefill_sweep(T), "device": "cuda", "scalar_gate": True})
    gs = inp["g"][..., 0].contiguous()
    o, fs = kda.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], gs, inp["beta"], initial_state=inp["s0"])
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    eo, es = _check(o, fs, inp, torch.tensor(HEADS), _kda_ref)
    assert eo < TOL and es < TOL, (eo, es)


@pytest.mark.slow
@pytest.mark.parametrize("T", synth.PREFILL_SWEEP_T)
def test_dplr_sweep_sampled_heads(kda, T):
    inp = synth.dplr_inputs(**synth.prefill_sweep(T), device="cuda")
    o, fs = kda.dplr_chunk_fwd(*(inp[n] for n in ("q", "k", "v", "a", "b", "g", "beta")), initial_state=inp["s0"])
    torch.cuda.synchronize()
    assert kda.device_status() == 0

    def ref(a, s0):
        return oracle.dplr_recurrent(a["q"], a["k"], a["v"], a["g"], a["beta"], a["a"], a["b"], s0=s0)

    # the product-form DPLR oracle costs O(d^3) per token: one sampled head
    eo, es = _check(o, fs, inp, torch.tensor([HEADS[1]]), ref)
    assert eo < TOL and es < TOL, (eo, es)
