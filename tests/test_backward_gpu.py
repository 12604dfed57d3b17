"""kda_recurrent_bwd vs the oracle's reverse mode (fp64).

The kernel evaluates every reverse step in fp32 (as the decode path does), so
each gradient is held to relative L2 <= 1e-4 over the tensor, the decode bar;
bf16 inputs are compared on their exact upcast values."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import f64, rel_l2

pytestmark = pytest.mark.gpu
TOL = 1e-4
NAMES = ("dq", "dk", "dv", "dg", "dbeta", "ds0")


def run_both(kda, B, T, H, dtype, seed, scale=1.0, with_states=True):
    inp = synth.op_inputs(B=B, H=H, T=T, dtype=dtype, s0_std=0.02 if with_states else None, seed=seed)
    gen = torch.Generator().manual_seed(seed + 1)
    do = torch.randn(inp["q"].shape, generator=gen).to(dtype)
    dsT = torch.randn((B, H, 128, 128), generator=gen) if with_states else None
    d = {n: inp[n].cuda() for n in ("q", "k", "v", "g", "beta")}
    got = kda.recurrent_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], do.cuda(),
                            initial_state=None if inp["s0"] is None else inp["s0"].cuda(),
                            d_final_state=None if dsT is None else dsT.cuda(), scale=scale)
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    ref = oracle.kda_recurrent_backward(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]), f64(inp["beta"]),
                                        f64(do), s0=f64(inp["s0"]), ds_final=f64(dsT), scale=scale)
    errs = {n: rel_l2(f64(x), r) for n, x, r in zip(NAMES, got, ref)}
    print(f"B={B} T={T} H={H} {dtype}: " + " ".join(f"{n}={e:.1e}" for n, e in errs.items()))
    for n, x in zip(NAMES, got):
        assert np.isfinite(f64(x)).all(), n
    return errs


@pytest.mark.parametrize("B,T,H", [(1, 1, 1), (2, 7, 3), (1, 64, 2), (1, 65, 2), (2, 130, 3)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_backward_small(kda, B, T, H, dtype):
    errs = run_both(kda, B, T, H, dtype, seed=500 + T + B, scale=0.9)
    assert all(e < TOL for e in errs.values()), errs


def test_backward_without_states(kda):
    errs = run_both(kda, 2, 70, 2, torch.float32, seed=510, with_states=False)
    assert all(e < TOL for e in errs.values() if not np.isnan(e)), errs


def test_backward_1000_tokens(kda):
    errs = run_both(kda, 1, 1000, 2, torch.bfloat16, seed=511)
    assert all(e < TOL for e in errs.values()), errs


def test_backward_empty_sequence_passes_state_gradient(kda):
    B, H = 2, 3
    z = torch.zeros((B, 0, H, 128), device="cuda", dtype=torch.bfloat16)
    dsT = torch.randn((B, H, 128, 128), device="cuda")
    got = kda.recurrent_bwd(z, z, z, z.float(), torch.zeros((B, 0, H), device="cuda"), z, d_final_state=dsT)
    torch.cuda.synchronize()
    assert torch.equal(got[5], dsT)
