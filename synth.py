"""Seeded synthetic inputs for KDA, shared by the tests, the bench and smoke().

This module only draws random numbers in the shapes and distributions of the
workloads; it holds none of the operator's arithmetic.  Both the CUDA path and
the oracle receive the same post-cast tensors from here (the oracle upcasts
them to fp64).

Workloads (shapes follow the pages' measurements: batch 1 with 16 heads and
head dim 128 up to 64K tokens; large-batch decode; one packed-varlen layer):

* ``op_inputs``     q, k ~ N(0,1) L2-normalised per head; v ~ N(0,1);
                    beta = sigmoid(N(0,1)); log-gate g = -gate_scale*softplus(N(0,1))
                    per channel; optional initial state ~ N(0, s0_std^2).
                    Draw order: q, k, v, beta-logit, gate-x, S0 (all fp32, then cast).
* ``decode_state`` / ``decode_step_inputs``  the same distributions per step.
* ``layer_inputs``  x ~ N(0,1) bf16, weights ~ N(0, 0.02^2), RMSNorm weight ones,
                    8 packed sequences whose 7 cut points are distinct uniform
                    integers in [1, Ttot-1].
"""
from __future__ import annotations

import torch

D = 128

# The five workloads, named by what they are.
ORACLE_SIZED = dict(B=1, H=2, T=256, dtype=torch.float32, gate_scale=0.1, s0_std=None, seed=1)
PREFILL_4K = dict(B=1, H=16, T=4096, dtype=torch.bfloat16, gate_scale=0.1, s0_std=0.02, seed=2)
PREFILL_SWEEP_T = (8192, 16384, 32768, 65536)
DECODE_B256 = dict(B=256, H=32, steps=1000, s0_std=0.02, seed=4)
LAYER_65K = dict(d_model=2048, H=16, Ttot=65536, nseq=8, rank=128, seed=5)


def prefill_sweep(T: int) -> dict:
    return dict(B=1, H=16, T=T, dtype=torch.bfloat16, gate_scale=0.1, s0_std=0.02, seed=3 + T)


def _gen(seed: int, device) -> torch.Generator:
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return gen


def _unit_heads(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True)


def op_inputs(B, H, T, dtype=torch.bfloat16, gate_scale=0.1, s0_std=None, seed=0, device="cpu",
              cu_seqlens=None, scalar_gate=False, **_):
    """Operator inputs.  Dense [B,T,H,D] when cu_seqlens is None, else packed
    [1,T,H,D] with the given cu_seqlens (then B is the number of sequences).

    scalar_gate=True draws one gate value per (token, head) and broadcasts it
    over the channels (the Gated DeltaNet special case)."""
    gen = _gen(seed, device)
    BT = 1 if cu_seqlens is not None else B
    shp = (BT, T, H, D)
    q = _unit_heads(torch.randn(shp, generator=gen, device=device))
    k = _unit_heads(torch.randn(shp, generator=gen, device=device))
    v = torch.randn(shp, generator=gen, device=device)
    beta = torch.sigmoid(torch.randn((BT, T, H), generator=gen, device=device))
    if scalar_gate:
        gx = torch.randn((BT, T, H, 1), generator=gen, device=device).expand(shp).contiguous()
    else:
        gx = torch.randn(shp, generator=gen, device=device)
    g = -gate_scale * torch.nn.functional.softplus(gx)
    nseq = B if cu_seqlens is None else len(cu_seqlens) - 1
    s0 = None
    if s0_std is not None:
        s0 = s0_std * torch.randn((nseq, H, D, D), generator=gen, device=device)
    out = dict(q=q.to(dtype), k=k.to(dtype), v=v.to(dtype), g=g.float().contiguous(),
               beta=beta.float().contiguous(), s0=s0)
    if cu_seqlens is not None:
        out["cu_seqlens"] = torch.as_tensor(cu_seqlens, dtype=torch.int32, device=device)
    return out


def dplr_inputs(B, H, T, dtype=torch.bfloat16, gate_scale=0.1, s0_std=None, seed=0, device="cpu",
                cu_seqlens=None, **_):
    """Inputs of the untied DPLR recurrence S = (I - a b^T) Diag(e^g) S + beta k v^T:
    the KDA inputs of ``op_inputs`` (same seed, same draws) plus a = sqrt(beta) k and
    b = sqrt(beta) bh, with bh an independent unit vector per (token, head), drawn
    after everything else.  bh = k would give back KDA."""
    out = op_inputs(B, H, T, dtype=dtype, gate_scale=gate_scale, s0_std=s0_std, seed=seed, device=device,
                    cu_seqlens=cu_seqlens)
    gen = _gen(seed * 7919 + 17, device)
    bh = _unit_heads(torch.randn(out["q"].shape, generator=gen, device=device))
    sb = out["beta"].sqrt()[..., None]
    out["a"] = (sb * out["k"].float()).to(dtype)
    out["b"] = (sb * bh).to(dtype)
    return out


def random_cu_seqlens(Ttot: int, nseq: int, seed: int) -> list:
    """nseq packed sequences: nseq-1 distinct uniform cut points in [1, Ttot-1]."""
    gen = _gen(seed, "cpu")
    cuts = torch.randperm(Ttot - 1, generator=gen)[: nseq - 1] + 1
    cuts = sorted(int(c) for c in cuts)
    return [0] + cuts + [Ttot]


def decode_state(B, H, s0_std=0.02, seed=0, device="cpu"):
    gen = _gen(seed, device)
    return s0_std * torch.randn((B, H, D, D), generator=gen, device=device)


def decode_step_inputs(B, H, step, seed=0, device="cpu", dtype=torch.bfloat16, gate_scale=0.1):
    """One token per sequence for decode step ``step`` (its own seeded stream)."""
    gen = _gen(seed * 1000003 + step + 1, device)
    shp = (B, H, D)
    q = _unit_heads(torch.randn(shp, generator=gen, device=device))
    k = _unit_heads(torch.randn(shp, generator=gen, device=device))
    v = torch.randn(shp, generator=gen, device=device)
    beta = torch.sigmoid(torch.randn((B, H), generator=gen, device=device))
    g = -gate_scale * torch.nn.functional.softplus(torch.randn(shp, generator=gen, device=device))
    return dict(q=q.to(dtype), k=k.to(dtype), v=v.to(dtype), g=g.float().contiguous(), beta=beta.float().contiguous())


def layer_inputs(d_model=2048, H=16, Ttot=65536, nseq=8, rank=128, seed=5, device="cpu", std=0.02):
    """Input activations, random-init weights and the packed-sequence layout."""
    gen = _gen(seed, device)
    HD = H * D

    def w(*shape):
        return (std * torch.randn(shape, generator=gen, device=device)).to(torch.bfloat16)

    x = torch.randn((Ttot, d_model), generator=gen, device=device).to(torch.bfloat16)
    W = dict(
        W_q=w(HD, d_model), W_k=w(HD, d_model), W_v=w(HD, d_model),
        W_adown=w(rank, d_model), W_gdown=w(rank, d_model), W_b=w(H, d_model),
        W_aup=w(HD, rank), W_gup=w(HD, rank),
        conv_q=w(HD, 4), conv_k=w(HD, 4), conv_v=w(HD, 4),
        norm_w=torch.ones(D, device=device, dtype=torch.float32),
        W_o=w(d_model, HD),
    )
    cu = random_cu_seqlens(Ttot, nseq, seed)
    return x, W, cu
