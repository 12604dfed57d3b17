"""The layer's fixed-size cache: kda_layer_fwd's conv and recurrent state
outputs, and kda_layer_decode continuing the sequences from them.

Each sequence is run by the fp64 oracle layer in one pass over all its tokens
(prompt, then the decoded tokens); the GPU runs a prefill and then decode calls
from the cache.  Tolerances as in test_layer_gpu.py: relative L2 1e-2 on y and on
the state."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import f64, rel_l2

pytestmark = pytest.mark.gpu
TOL_Y = 1e-2
TOL_S = 1e-2


def setup(d_model, H, rank, total, seed):
    x, W, _ = synth.layer_inputs(d_model=d_model, H=H, Ttot=total, nseq=1, rank=rank, seed=seed)
    import gated_delta_rule_123_b200 as kda
    packed = kda.pack_layer_weights({n: t.to(torch.device("cuda")) for n, t in W.items()})
    return x, W, packed


def oracle_seq(x_rows, W, H, s0):
    return oracle.kda_layer(f64(x_rows), {n: f64(t) for n, t in W.items()}, [0, x_rows.shape[0]], H,
                            s0=None if s0 is None else f64(s0)[None])


@pytest.mark.parametrize("prompt_lens,steps", [([37, 1, 100], [5, 1, 3]), ([0, 2, 64], [4, 4])])
def test_prefill_then_decode(kda, prompt_lens, steps):
    d_model, H, rank = 256, 2, 32
    N = len(prompt_lens)
    P = sum(prompt_lens)
    total = P + N * sum(steps)
    x, W, packed = setup(d_model, H, rank, total, seed=41 + P)
    dev = torch.device("cuda")
    S0 = 0.02 * torch.randn((N, H, 128, 128), generator=torch.Generator().manual_seed(41))
    cu = np.concatenate([[0], np.cumsum(prompt_lens)]).astype(np.int32)
    xp = x[:P]
    y_pre, S, C = kda.layer_fwd(xp.to(dev), packed, torch.tensor(cu, device=dev), initial_state=S0.to(dev),
                                output_conv_state=True)
    ys, off = [], P
    for T in steps:
        xd = x[off:off + N * T].reshape(N, T, d_model)
        off += N * T
        ys.append((xd, kda.layer_decode(xd.to(dev).contiguous(), packed, C, S)))
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    for n in range(N):
        rows = [xp[cu[n]:cu[n + 1]]] + [xd[n] for xd, _ in ys]
        y_ref, s_ref = oracle_seq(torch.cat(rows, 0), W, H, S0[n])
        got = [f64(y_pre)[cu[n]:cu[n + 1]]] + [f64(yd)[n] for _, yd in ys]
        y_got = np.concatenate(got, 0)
        ey, es = rel_l2(y_got, y_ref), rel_l2(f64(S)[n], s_ref[0])
        ey_dec = rel_l2(y_got[prompt_lens[n]:], y_ref[prompt_lens[n]:])
        print(f"seq {n}: prompt {prompt_lens[n]}: rel-L2 y={ey:.2e} (decoded part {ey_dec:.2e}) state={es:.2e}")
        assert ey < TOL_Y and ey_dec < TOL_Y and es < TOL_S


def test_conv_cache_contents(kda):
    """conv_state_out holds the last three q/k/v projections of each sequence,
    oldest first, with zero rows before a sequence's first token."""
    d_model, H, rank = 128, 1, 16
    lens = [5, 2, 0, 3]
    x, W, packed = setup(d_model, H, rank, sum(lens), seed=42)
    dev = torch.device("cuda")
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    _, _, C = kda.layer_fwd(x.to(dev), packed, torch.tensor(cu, device=dev), output_conv_state=True)
    torch.cuda.synchronize()
    Wqkv = np.concatenate([f64(W["W_q"]), f64(W["W_k"]), f64(W["W_v"])], 0)
    z = f64(x) @ Wqkv.T
    Cn = f64(C)
    for n, L in enumerate(lens):
        for j in range(3):
            p = cu[n + 1] - 3 + j
            if p < cu[n]:
                assert np.all(Cn[n, j] == 0.0), (n, j)
            else:
                assert rel_l2(Cn[n, j], z[p]) < 1e-2, (n, j)


def test_chunked_prefill_through_the_cache(kda):
    """A prompt split in two kda_layer_fwd calls (conv and recurrent state
    carried through the cache) matches the oracle over the whole prompt."""
    d_model, H, rank = 256, 2, 32
    lens_a, lens_b = [50, 2, 130], [70, 1, 2]
    N = 3
    total = sum(lens_a) + sum(lens_b)
    x, W, packed = setup(d_model, H, rank, total, seed=43)
    dev = torch.device("cuda")
    cu_a = np.concatenate([[0], np.cumsum(lens_a)]).astype(np.int32)
    cu_b = np.concatenate([[0], np.cumsum(lens_b)]).astype(np.int32)
    xa, xb = x[:sum(lens_a)], x[sum(lens_a):]
    ya, S, C = kda.layer_fwd(xa.to(dev), packed, torch.tensor(cu_a, device=dev), output_conv_state=True)
    yb, S2, C2 = kda.layer_fwd(xb.to(dev), packed, torch.tensor(cu_b, device=dev), initial_state=S,
                               conv_state_in=C, output_conv_state=True)
    torch.cuda.synchronize()
    for n in range(N):
        rows = torch.cat([xa[cu_a[n]:cu_a[n + 1]], xb[cu_b[n]:cu_b[n + 1]]], 0)
        y_ref, s_ref = oracle_seq(rows, W, H, None)
        y_got = np.concatenate([f64(ya)[cu_a[n]:cu_a[n + 1]], f64(yb)[cu_b[n]:cu_b[n + 1]]], 0)
        ey, es = rel_l2(y_got, y_ref), rel_l2(f64(S2)[n], s_ref[0])
        print(f"seq {n}: rel-L2 y={ey:.2e} state={es:.2e}")
        assert ey < TOL_Y and es < TOL_S
