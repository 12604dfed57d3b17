"""kda_chunk_fwd vs the fp64 oracle recurrence.

Tolerance (from the operator's precision: bf16 tensor-core operands, fp32
accumulation and fp32 state): relative L2 error <= 1e-2 on o and on the final
state, over the whole tensor.  The oracle's fp64 o is compared directly (the
GPU rounds o to bf16 once, ~2e-3 relative)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import f64, rel_l2

pytestmark = pytest.mark.gpu
TOL = 1e-2


def run_both(kda, inp, scale=1.0, l2=False, heads=None):
    q, k, v, g, beta = (inp[n] for n in ("q", "k", "v", "g", "beta"))
    cu = inp.get("cu_seqlens")
    s0 = inp.get("s0")
    o, fs = kda.chunk_fwd(q.cuda(), k.cuda(), v.cuda(), g.cuda(), beta.cuda(),
                          initial_state=None if s0 is None else s0.cuda(),
                          cu_seqlens=None if cu is None else cu.cuda(), scale=scale, l2norm_qk=l2)
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    if heads is not None:  # compare a subset of heads (sliced before leaving the device)
        hs = torch.as_tensor(heads) if isinstance(heads, list) else torch.arange(q.shape[2])[heads]
        hs = hs.to(q.device)
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


def test_oracle_sized_fp32(kda):
    """B=1, H=2, T=256 fp32, zero initial state (the oracle-sized workload)."""
    inp = synth.op_inputs(**synth.ORACLE_SIZED)
    eo, es = run_both(kda, inp)
    assert eo < TOL and es < TOL, (eo, es)


@pytest.mark.parametrize("B,T,H", [(1, 64, 1), (1, 1, 2), (2, 63, 2), (1, 65, 3), (2, 200, 3), (3, 130, 5)])
def test_small_shapes_bf16_with_state(kda, B, T, H):
    inp = synth.op_inputs(B=B, H=H, T=T, s0_std=0.02, seed=100 + T)
    eo, es = run_both(kda, inp, scale=0.9)
    assert eo < TOL and es < TOL, (eo, es)


def test_no_segment_scan_path(kda):
    """Enough (sequence, head) pairs that every CTA runs a whole sequence."""
    inp = synth.op_inputs(B=4, H=40, T=300, s0_std=0.02, seed=7)
    eo, es = run_both(kda, inp, heads=slice(0, 40, 7))
    assert eo < TOL and es < TOL, (eo, es)


def test_strong_decay_exact_fallback(kda):
    """Gates ~20x stronger: the in-chunk decay range exceeds the factored
    path's bound, so chunks take the exact fallback."""
    inp = synth.op_inputs(B=1, H=2, T=257, gate_scale=3.0, s0_std=0.02, seed=8)
    eo, es = run_both(kda, inp)
    assert eo < TOL and es < TOL, (eo, es)


def test_mixed_decay_strength(kda):
    inp = synth.op_inputs(B=1, H=2, T=512, gate_scale=1.0, s0_std=0.02, seed=9)
    inp["g"][:, 200:300] *= 4.0
    eo, es = run_both(kda, inp)
    assert eo < TOL and es < TOL, (eo, es)


def test_scalar_gate_gdn_case(kda):
    inp = synth.op_inputs(B=1, H=4, T=333, s0_std=0.02, seed=10, scalar_gate=True)
    eo, es = run_both(kda, inp)
    assert eo < TOL and es < TOL, (eo, es)


def test_l2norm_in_kernel(kda):
    inp = synth.op_inputs(B=1, H=2, T=150, s0_std=0.02, seed=12)
    inp["q"] = (inp["q"].float() * 4.0).bfloat16()
    inp["k"] = (inp["k"].float() * 0.3).bfloat16()
    eo, es = run_both(kda, inp, l2=True)
    assert eo < TOL and es < TOL, (eo, es)


def test_varlen_with_empty_and_short_sequences(kda):
    cu = [0, 0, 5, 69, 70, 70, 300, 301, 600]
    inp = synth.op_inputs(B=len(cu) - 1, H=3, T=cu[-1], s0_std=0.02, seed=13, cu_seqlens=cu)
    eo, es = run_both(kda, inp)
    assert eo < TOL and es < TOL, (eo, es)


def test_varlen_mixes_whole_and_segmented_sequences(kda):
    """Packed sequences of 100, 6000, 50 and 5850 tokens with H=4: 16 pairs, so the
    plan cuts sequences into 6-chunk segments.  The two long sequences run through
    the map / combine / light-output path in 16 segments each, while the two short
    ones run whole in the first launch.  Parity against the oracle, and the same bits
    whether the chunk products are exported or recomputed."""
    cu = [0, 100, 6100, 6150, 12000]
    H = 4
    assert kda.chunk_fwd_segments(1, cu[-1], H, len(cu) - 1) == (6 * 64, 6 * 64)
    inp = synth.op_inputs(B=len(cu) - 1, H=H, T=cu[-1], s0_std=0.02, seed=18, cu_seqlens=cu)
    eo, es = run_both(kda, inp)
    assert eo < TOL and es < TOL, (eo, es)
    d = [inp[n].cuda() for n in ("q", "k", "v", "g", "beta")]
    cu_d, s0 = inp["cu_seqlens"].cuda(), inp["s0"].cuda()
    lib = kda.lib()
    nseq = len(cu) - 1
    full = lib.kda_chunk_fwd_workspace(1, cu[-1], H, nseq, 0, 0)
    small = lib.kda_chunk_fwd_workspace_min(1, cu[-1], H, nseq, 0, 0)
    assert small < full
    res = [kda.chunk_fwd(*d, initial_state=s0, cu_seqlens=cu_d,
                         workspace=torch.empty(nbytes, device="cuda", dtype=torch.uint8)) for nbytes in (full, small)]
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])


# 8 packed sequences of 100 ... 5000 tokens (2 to 79 chunks) x 16 heads: 128 pairs,
# too many for the uniform segment plan, so the device cuts the lengths itself.
BALANCED_CU = [0, 100, 5100, 5164, 7164, 7165, 11165, 11900, 12000]


def test_balanced_plan_cuts_long_packed_sequences(kda):
    """The device plan keeps the short sequences whole and cuts the long ones at a
    common target length: segment 0 runs its output in the first launch from the
    initial state, the later segments a map there and their output in the second
    launch, and sequences of three or more segments chain their maps through the
    combine pass.  Parity against the oracle on four heads; the same bits whether
    the later segments read back the exported chunk products (the full workspace)
    or recompute them (any smaller workspace that still holds the per-segment
    states); the minimal workspace runs unsegmented, within rounding."""
    cu, H = BALANCED_CU, 16
    T, nseq = cu[-1], len(cu) - 1
    assert kda.chunk_fwd_segments(1, T, H, nseq) == (-1, -1)
    inp = synth.op_inputs(B=nseq, H=H, T=T, s0_std=0.02, seed=31, cu_seqlens=cu)
    eo, es = run_both(kda, inp, heads=[0, 5, 10, 15])
    assert eo < TOL and es < TOL, (eo, es)
    d = [inp[n].cuda() for n in ("q", "k", "v", "g", "beta")]
    cu_d, s0 = inp["cu_seqlens"].cuda(), inp["s0"].cuda()
    lib = kda.lib()
    full = lib.kda_chunk_fwd_workspace(1, T, H, nseq, 0, 0)
    small = lib.kda_chunk_fwd_workspace_min(1, T, H, nseq, 0, 0)
    assert small < full - 256
    res, plans = [], []
    for nbytes in (full, full - 256, small):
        ws = torch.empty(nbytes, device="cuda", dtype=torch.uint8)
        res.append(kda.chunk_fwd(*d, initial_state=s0, cu_seqlens=cu_d, workspace=ws))
        plans.append(kda.chunk_fwd_plan(ws, 1, T, H, nseq))
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])
    assert plans[0] == plans[1] and len(plans[2]) == nseq  # the minimal workspace: one item per sequence
    for a, b in zip(res[0], res[2]):
        assert rel_l2(f64(a), f64(b)) < 5e-3
    plan = plans[0]
    # the segments tile every sequence in order, on chunk boundaries
    for n in range(nseq):
        segs = [r for r in plan if r[0] == n]
        assert segs[0][1] == cu[n] and segs[-1][2] == cu[n + 1]
        assert [r[3] for r in segs] == list(range(len(segs))) and all(r[4] == len(segs) for r in segs)
        for a, b in zip(segs, segs[1:]):
            assert a[2] == b[1] and (b[1] - cu[n]) % 64 == 0 and b[1] < b[2]
    G = {r[0]: r[4] for r in plan}
    print("segments per sequence:", [G[n] for n in range(nseq)])
    assert G[1] >= 3 and G[0] == 1 and G[4] == 1  # the 5000-token one chains; 100 and 1 token stay whole


def test_balanced_plan_with_empty_sequences_and_no_initial_state(kda):
    cu = [0, 0, 3000, 3000, 3001, 4500, 4500, 9000, 9100]
    inp = synth.op_inputs(B=len(cu) - 1, H=16, T=cu[-1], s0_std=None, seed=32, cu_seqlens=cu)
    assert kda.chunk_fwd_segments(1, cu[-1], 16, len(cu) - 1) == (-1, -1)
    eo, es = run_both(kda, inp, heads=[3, 12])
    assert eo < TOL and es < TOL, (eo, es)


def test_balanced_plan_fp32_inputs_with_l2norm(kda):
    """fp32 q, k, v (rounded to bf16 operands, fp32 o) normalised in the kernel, on a
    packed call the device plan cuts (one 38-chunk sequence among short ones)."""
    cu = [0, 100, 2500, 2600, 2700, 2701, 2800, 2900, 3000]
    assert kda.chunk_fwd_segments(1, cu[-1], 16, len(cu) - 1) == (-1, -1)
    inp = synth.op_inputs(B=len(cu) - 1, H=16, T=cu[-1], dtype=torch.float32, s0_std=0.02, seed=34, cu_seqlens=cu)
    inp["q"] = inp["q"] * 3.0
    inp["k"] = inp["k"] * 0.5
    eo, es = run_both(kda, inp, l2=True, heads=[2, 9])
    assert eo < TOL and es < TOL, (eo, es)


def test_final_state_only_and_zero_state(kda):
    inp = synth.op_inputs(B=2, H=2, T=100, s0_std=None, seed=14)
    eo, es = run_both(kda, inp)
    assert eo < TOL and es < TOL, (eo, es)


def test_deterministic_bits(kda):
    inp = synth.op_inputs(B=1, H=2, T=700, s0_std=0.02, seed=15)
    a = [kda.chunk_fwd(*(inp[n].cuda() for n in ("q", "k", "v", "g", "beta")), initial_state=inp["s0"].cuda())
         for _ in range(2)]
    assert torch.equal(a[0][0], a[1][0]) and torch.equal(a[0][1], a[1][1])


def test_prefill_4k_full(kda):
    """B=1, H=16, T=4096 bf16 with a random initial state: every head."""
    inp = synth.op_inputs(**synth.PREFILL_4K)
    eo, es = run_both(kda, inp)
    assert eo < TOL and es < TOL, (eo, es)


@pytest.mark.slow
def test_prefill_64k_sampled_heads(kda):
    """B=1, H=16, T=65536 (the length sweep's largest point), in the launch
    configuration the bench times; the oracle checks heads 0, 5, 11 and 15."""
    inp = synth.op_inputs(**synth.prefill_sweep(65536), device="cuda")
    eo, es = run_both(kda, inp, heads=[0, 5, 11, 15])
    assert eo < TOL and es < TOL, (eo, es)


@pytest.mark.parametrize("scalar_gate", [False, True])
def test_both_segmented_schedules_give_identical_bits(kda, scalar_gate):
    """With the full workspace each segment's output pass reads back the chunk
    products its map pass exported; with the minimal one it recomputes them.  The
    same values go through the same MMAs either way."""
    B, T, H = 1, 3000, 16
    inp = synth.op_inputs(B=B, H=H, T=T, s0_std=0.02, seed=16, scalar_gate=scalar_gate)
    d = {n: inp[n].cuda() for n in ("q", "k", "v", "g", "beta")}
    if scalar_gate:
        d["g"] = d["g"][..., 0].contiguous()
    fn = kda.gdn_chunk_fwd if scalar_gate else kda.chunk_fwd
    lib = kda.lib()
    full = lib.kda_chunk_fwd_workspace(B, T, H, 0, 0, 0)
    small = lib.kda_chunk_fwd_workspace_min(B, T, H, 0, 0, 0)
    assert kda.chunk_fwd_segments(B, T, H)[0] > 0 and small < full
    res = []
    for nbytes in (full, small):
        ws = torch.empty(nbytes, device="cuda", dtype=torch.uint8)
        res.append(fn(*(d[n] for n in ("q", "k", "v", "g", "beta")), initial_state=inp["s0"].cuda(), workspace=ws))
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])


def test_cuda_graph_replay_matches_eager_and_traces_launches(kda):
    """A segmented call captured into a CUDA graph (as the benchmark times it) gives
    the eager call's bits on replay, and trace events set during the capture time
    each of its launches."""
    B, T, H = 1, 3000, 16
    inp = synth.op_inputs(B=B, H=H, T=T, s0_std=0.02, seed=17)
    d = [inp[n].cuda() for n in ("q", "k", "v", "g", "beta")]
    s0 = inp["s0"].cuda()
    assert kda.chunk_fwd_segments(B, T, H)[0] > 0
    ws = torch.empty(kda.chunk_fwd_workspace_bytes(B, T, H), device="cuda", dtype=torch.uint8)
    o_ref, fs_ref = kda.chunk_fwd(*d, initial_state=s0, workspace=ws)
    o, fs = torch.empty_like(o_ref), torch.empty_like(fs_ref)
    torch.cuda.synchronize()
    events = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    for e in events:  # created outside the capture
        e.record()
    graph = torch.cuda.CUDAGraph()
    try:
        with torch.cuda.graph(graph):
            kda.set_trace_events(events)
            kda.chunk_fwd(*d, initial_state=s0, out=o, final_state=fs, workspace=ws)
    finally:
        kda.set_trace_events(None)
    o.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    assert torch.equal(o, o_ref) and torch.equal(fs, fs_ref)
    times = [events[i].elapsed_time(events[i + 1]) for i in range(4)]
    assert all(t >= 0 for t in times) and times[1] > 0 and times[3] > 0, times
