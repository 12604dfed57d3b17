"""kda_linear_bf16 (the layer's projection GEMM on the tensor cores) against a
float64 product of the same bf16 values on the CPU.

The projections of "Kimi Linear: An Expressive, Efficient Attention
Architecture" ("Neural Parameterization") are plain bias-free linear maps
y = x W^T; the reference is that definition in float64.  The kernel
accumulates in fp32 and rounds y to bf16 once (relative 2^-9 per element), so
the bar is relative L2 <= 2e-3 over the output and an elementwise error below
2^-7 of the largest |y|.  Shapes cover tails in M, N (a last tile narrower than
256 columns issues narrower MMAs) and K (not a multiple of 64), the layer's
input projection (N = 3*2048 + 2*128 + 16 = 6416, K = 2048) and its output
projection; the full 65536-row launch is checked on sampled rows."""
import numpy as np
import pytest
import torch

from helpers import f64, rel_l2

pytestmark = pytest.mark.gpu


def _rand(shape, gen, std=1.0):
    return (std * torch.randn(shape, generator=gen)).to(torch.bfloat16)


def _check(y, x, W, rows=None):
    xs = x if rows is None else x[rows]
    ref = f64(xs) @ f64(W).T
    got = f64(y if rows is None else y[rows])
    e = rel_l2(got, ref)
    emax = np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30)
    print(f"rel-L2 {e:.2e}  max err / max|y| {emax:.2e}")
    assert e < 2e-3 and emax < 2 ** -7, (e, emax)


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (1, 16, 8), (300, 834, 256), (257, 200, 136),
                                   (1000, 6416, 2048), (777, 2048, 2048), (4096, 2048, 128)])
def test_linear_matches_float64_product(kda, M, N, K):
    gen = torch.Generator().manual_seed(M * 7 + N * 3 + K)
    x, W = _rand((M, K), gen), _rand((N, K), gen, 0.02)
    y = kda.linear(x.cuda(), W.cuda())
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    _check(y.cpu(), x, W)


def test_linear_row_strides_and_determinism(kda):
    """Operands inside larger row-major buffers (row strides above the row length),
    as the layer reads the low-rank slices of its input projection; same bits on
    a second call."""
    gen = torch.Generator().manual_seed(5)
    M, N, K = 500, 384, 128
    xb, Wb = _rand((M, K + 40), gen), _rand((N, K + 8), gen, 0.02)
    x, W = xb[:, 24:24 + K], Wb[:, :K]
    lib = kda.lib()
    xd, Wd = xb.cuda(), Wb.cuda()
    outs = []
    for _ in range(2):
        yb = torch.full((M, N + 16), float("nan"), device="cuda", dtype=torch.bfloat16)
        import ctypes
        rc = lib.kda_linear_bf16(ctypes.c_void_p(xd.data_ptr() + 24 * 2), K + 40, ctypes.c_void_p(Wd.data_ptr()), K + 8,
                                 ctypes.c_void_p(yb.data_ptr()), N + 16, M, N, K,
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == 0, lib.kda_last_error()
        torch.cuda.synchronize()
        outs.append(yb)
    assert torch.equal(outs[0][:, :N], outs[1][:, :N])
    assert torch.isnan(outs[0][:, N:].float()).all()  # nothing written past the N columns
    _check(outs[0][:, :N].cpu(), x, W)


@pytest.mark.slow
def test_linear_full_size_input_projection_sampled_rows(kda):
    """The layer's input projection at full size, 65536 x 6416 x 2048, in one
    launch; 96 sampled rows (first, last and spread) against float64."""
    gen = torch.Generator(device="cuda").manual_seed(6)
    M, N, K = 65536, 6416, 2048
    x = torch.randn((M, K), generator=gen, device="cuda").to(torch.bfloat16)
    W = (0.02 * torch.randn((N, K), generator=gen, device="cuda")).to(torch.bfloat16)
    y = kda.linear(x, W)
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    rows = torch.cat([torch.arange(32), torch.arange(M - 32, M), torch.randperm(M, generator=torch.Generator().manual_seed(7))[:32]])
    _check(y[rows.cuda()].cpu(), x[rows.cuda()].cpu(), W.cpu())


def test_linear_rejects_bad_arguments(kda):
    lib = kda.lib()
    import ctypes
    x = torch.zeros((64, 64), device="cuda", dtype=torch.bfloat16)
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = ctypes.c_void_p(x.data_ptr())
    assert lib.kda_linear_bf16(p, 64, p, 64, None, 64, 64, 64, 64, s) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_linear_bf16(p, 60, p, 64, p, 64, 64, 64, 60, s) == kda.KDA_ERR_INVALID_ARG  # stride not 16 B
    assert lib.kda_linear_bf16(p, 64, p, 64, p, 64, 64, 64, 64, s) == kda.KDA_ERR_INVALID_ARG  # y aliases x
