"""kda_recurrent_fwd (fused recurrent segments) vs the fp64 oracle recurrence.

The kernel computes in fp32 on CUDA cores, so the state is held to the decode
bar (relative L2 <= 1e-4 after the segment); o is held to 1e-4 for fp32 inputs
and, for bf16 output, to 1e-2 against the oracle rounded to bf16 once."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import f64, rel_l2

pytestmark = pytest.mark.gpu


def oracle_segment(inp, S, scale=1.0, l2=False):
    q, k = f64(inp["q"]), f64(inp["k"])
    if l2:
        q = q / np.sqrt((q * q).sum(-1, keepdims=True) + 1e-6)
        k = k / np.sqrt((k * k).sum(-1, keepdims=True) + 1e-6)
    return oracle.kda_recurrent(q, k, f64(inp["v"]), f64(inp["g"]), f64(inp["beta"]), s0=S, scale=scale)


def check(kda, B, T, H, dtype, seed, scale=1.0, l2=False, gate_scale=0.1):
    inp = synth.op_inputs(B=B, H=H, T=T, dtype=dtype, gate_scale=gate_scale, seed=seed)
    S = synth.decode_state(B, H, seed=seed).cuda()
    S0 = f64(S)
    d = {n: inp[n].cuda() for n in ("q", "k", "v", "g", "beta")}
    if l2:
        d["q"] = (d["q"].float() * 2.5).to(dtype)
        d["k"] = (d["k"].float() * 0.4).to(dtype)
    o = kda.recurrent_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S, scale=scale, l2norm_qk=l2)
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    o_ref, S_ref = oracle_segment(d, S0, scale=scale, l2=l2)
    es = rel_l2(f64(S), S_ref)
    if dtype == torch.bfloat16:
        eo = rel_l2(f64(o), torch.tensor(o_ref).bfloat16().double().numpy())
        tol_o = 1e-2
    else:
        eo = rel_l2(f64(o), o_ref)
        tol_o = 1e-4
    print(f"B={B} T={T} H={H} {dtype}: rel-L2 o={eo:.2e} state={es:.2e}")
    assert eo < tol_o and es < 1e-4, (eo, es)


@pytest.mark.parametrize("B,T,H", [(1, 1, 1), (2, 7, 3), (4, 64, 8), (3, 100, 2), (1, 2, 5)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_recurrent_segments(kda, B, T, H, dtype):
    check(kda, B, T, H, dtype, seed=300 + T + B, scale=0.9)


def test_recurrent_l2norm_and_strong_decay(kda):
    check(kda, 2, 33, 3, torch.float32, seed=310, l2=True, gate_scale=3.0)


def test_recurrent_one_token_matches_decode_step(kda):
    B, H = 4, 6
    inp = {k: v.cuda() for k, v in synth.decode_step_inputs(B, H, 0, seed=311, dtype=torch.float32).items()}
    S1 = synth.decode_state(B, H, seed=311).cuda()
    S2 = S1.clone()
    o1 = kda.decode_step(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S1)
    seg = {n: t.unsqueeze(1).contiguous() for n, t in inp.items()}  # [B,1,H,...]
    o2 = kda.recurrent_fwd(seg["q"], seg["k"], seg["v"], seg["g"], seg["beta"], S2)
    torch.cuda.synchronize()
    assert rel_l2(f64(o2[:, 0]), f64(o1)) < 1e-6 and rel_l2(f64(S2), f64(S1)) < 1e-6


def test_recurrent_split_is_bit_exact(kda):
    """Running [0, a) then [a, T) equals running [0, T): the fp32 state crosses
    calls unchanged."""
    B, T, H, a = 2, 50, 3, 19
    inp = {n: t.cuda() for n, t in synth.op_inputs(B=B, H=H, T=T, seed=312).items() if t is not None and n != "s0"}
    S1 = synth.decode_state(B, H, seed=312).cuda()
    S2 = S1.clone()
    o1 = kda.recurrent_fwd(*(inp[n] for n in ("q", "k", "v", "g", "beta")), S1)
    parts = [{n: t[:, lo:hi].contiguous() for n, t in inp.items()} for lo, hi in ((0, a), (a, T))]
    o2 = torch.cat([kda.recurrent_fwd(*(p[n] for n in ("q", "k", "v", "g", "beta")), S2) for p in parts], dim=1)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_recurrent_continues_a_chunked_prefill(kda):
    """Prefill 500 tokens with kda_chunk_fwd, then 40 tokens with
    kda_recurrent_fwd from its final state (the pages' prompt-then-decode
    split); both parts vs one oracle run over all 540 tokens."""
    B, H, T, P = 1, 4, 540, 500
    inp = synth.op_inputs(B=B, H=H, T=T, s0_std=0.02, seed=313)
    d = {n: inp[n].cuda() for n in ("q", "k", "v", "g", "beta")}
    pre = {n: t[:, :P].contiguous() for n, t in d.items()}
    seg = {n: t[:, P:].contiguous() for n, t in d.items()}
    o1, S = kda.chunk_fwd(*(pre[n] for n in ("q", "k", "v", "g", "beta")), initial_state=inp["s0"].cuda())
    o2 = kda.recurrent_fwd(*(seg[n] for n in ("q", "k", "v", "g", "beta")), S)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_segment(d, f64(inp["s0"]))
    eo = rel_l2(f64(torch.cat([o1, o2], dim=1)), o_ref)
    es = rel_l2(f64(S), S_ref)
    print(f"prefill+segment: rel-L2 o={eo:.2e} state={es:.2e}")
    assert eo < 1e-2 and es < 1e-2


def test_recurrent_b256_h32_t16_sampled_heads(kda):
    """The decode workload's shape with 16-token segments: B=256, H=32, T=16;
    the oracle checks 5 sampled (sequence, head) pairs."""
    B, H, T = 256, 32, 16
    inp = synth.op_inputs(B=B, H=H, T=T, seed=314, device="cuda")
    S = synth.decode_state(B, H, seed=314, device="cuda")
    S0 = S.clone()
    o = kda.recurrent_fwd(*(inp[n] for n in ("q", "k", "v", "g", "beta")), S)
    torch.cuda.synchronize()
    for b, h in ((0, 0), (17, 5), (128, 31), (200, 9), (255, 16)):
        sub = {n: inp[n][b:b + 1, :, h:h + 1] for n in ("q", "k", "v", "g", "beta")}
        o_ref, S_ref = oracle_segment(sub, f64(S0[b:b + 1, h:h + 1]))
        eo = rel_l2(f64(o[b:b + 1, :, h:h + 1]), torch.tensor(o_ref).bfloat16().double().numpy())
        es = rel_l2(f64(S[b:b + 1, h:h + 1]), S_ref)
        assert eo < 1e-2 and es < 1e-4, (b, h, eo, es)
