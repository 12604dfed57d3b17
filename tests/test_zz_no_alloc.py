"""kda_chunk_fwd_noalloc: the entry point for callers that cannot allocate.

Callers such as a plugin inside a runtime that owns all device memory, or a
serving loop that must not call cudaMalloc mid-step, cannot hand the library a
workspace; this entry point takes its scratch from a static device array
instead.  Here it is called through the C ABI (ctypes, no Python wrapper) and
must reproduce kda_chunk_fwd (which uses a caller workspace) on two calls in a
row.  The same kernels run on the same values, so the outputs must be
bit-identical (a stricter bar than the chunk tests' relative L2 of 1e-2
against the oracle).  This file is collected last.
"""
import ctypes

import pytest
import torch

import synth
from helpers import f64, rel_l2

pytestmark = pytest.mark.gpu


def _noalloc(kda):
    lib = ctypes.CDLL(kda.LIB_PATH)
    fn = lib.kda_chunk_fwd_noalloc
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fn.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
    fn.restype = i
    return fn


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("case", ["dense_4k_scan", "varlen", "varlen_balanced"])
def test_noalloc_matches_workspace_entry_point_two_calls(kda, case):
    """varlen_balanced: 8 packed sequences x 8 heads, one of them 38 chunks long, so the
    device plan cuts it; the full workspace (product images and per-segment states,
    ~50 MB) fits the static array, so both entry points run the same cuts."""
    fn = _noalloc(kda)
    dev = torch.device("cuda")
    if case == "dense_4k_scan":
        inp = synth.op_inputs(**synth.PREFILL_4K, device=dev)
        cu = None
    elif case == "varlen":
        cuv = [0, 5, 69, 70, 300, 777]
        inp = synth.op_inputs(B=len(cuv) - 1, H=3, T=cuv[-1], s0_std=0.02, seed=31, cu_seqlens=cuv, device=dev)
        cu = inp["cu_seqlens"]
    else:
        cuv = [0, 100, 2500, 2600, 2700, 2701, 2800, 2900, 3000]
        assert kda.chunk_fwd_segments(1, cuv[-1], 8, len(cuv) - 1) == (-1, -1)
        assert kda.chunk_fwd_workspace_bytes(1, cuv[-1], 8, len(cuv) - 1) <= 64 << 20
        inp = synth.op_inputs(B=len(cuv) - 1, H=8, T=cuv[-1], s0_std=0.02, seed=35, cu_seqlens=cuv, device=dev)
        cu = inp["cu_seqlens"]
    q, k, v, g, beta, s0 = (inp[n] for n in ("q", "k", "v", "g", "beta", "s0"))
    B, T, H, _ = q.shape
    nseq = 0 if cu is None else cu.numel() - 1
    o_ref, fs_ref = kda.chunk_fwd(q, k, v, g, beta, initial_state=s0, cu_seqlens=cu)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        o = torch.full_like(q, float("nan"))
        fs = torch.full_like(fs_ref, float("nan"))
        rc = fn(_p(q), _p(k), _p(v), _p(g), _p(beta), _p(s0), _p(fs), _p(o), _p(cu), nseq, B, T, H, kda.KDA_BF16,
                1.0, 0, stream)
        assert rc == kda.KDA_OK, kda.lib().kda_last_error()
        torch.cuda.synchronize()
        assert kda.device_status() == 0
        assert torch.isfinite(o.float()).all() and torch.isfinite(fs).all()
        assert torch.equal(o, o_ref), (call, rel_l2(f64(o), f64(o_ref)))
        assert torch.equal(fs, fs_ref), (call, rel_l2(f64(fs), f64(fs_ref)))


def test_noalloc_rejects_calls_beyond_its_static_scratch(kda):
    fn = _noalloc(kda)
    # fp32 inputs at B=1, H=16, T=65536 need bf16 copies of q, k, v in scratch (~800 MB):
    # far beyond the 64 MiB array, so the call is rejected before any launch
    B, T, H = 1, 65536, 16
    assert kda.chunk_fwd_workspace_bytes(B, T, H, 0, kda.KDA_FP32) > 64 << 20
    rc = fn(None, None, None, None, None, None, None, None, None, 0, B, T, H, kda.KDA_FP32, 1.0, 0, None)
    assert rc == kda.KDA_ERR_UNSUPPORTED
    assert b"scratch" in kda.lib().kda_last_error()
