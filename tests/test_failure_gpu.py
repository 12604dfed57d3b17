"""Failure detection on the GPU without a fault: a bounded device-side wait
that gives up.

The chunk kernels wait on mbarriers for their TMA loads and MMAs; every such
wait is bounded.  Here the host makes the loader skip one chunk's q/k/g load
(``kda_debug_fault_injection``), with the wait bound lowered to 2^22 cycles
(about 2 ms).  The consumer's wait then runs out: the kernel must record
KDA_ERR_TIMEOUT in the device status word, let its in-flight copies land,
free its tensor memory and exit -- no trap, no hang -- and the next call on the
same stream must run normally and match the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import f64, rel_l2

pytestmark = pytest.mark.gpu
TOL = 1e-2


def _oracle_check(inp, o, fs):
    o_ref, s_ref = oracle.kda_recurrent(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                                        f64(inp["beta"]), s0=f64(inp["s0"]))
    return rel_l2(f64(o), o_ref), rel_l2(f64(fs), s_ref)


@pytest.mark.parametrize("skip", [0, 2])
def test_skipped_load_times_out_cleanly_then_next_call_is_correct(kda, skip):
    # 64 (sequence, head) pairs: every CTA runs a whole 4-chunk sequence (no segment scan)
    B, T, H = 1, 256, 64
    assert kda.chunk_fwd_segments(B, T, H) == (0, 0)
    inp = synth.op_inputs(B=B, H=H, T=T, s0_std=0.02, seed=41)
    d = {n: inp[n].cuda() for n in ("q", "k", "v", "g", "beta", "s0")}
    assert kda.device_status() == kda.KDA_OK
    kda.debug_fault_injection(wait_limit_cycles=1 << 22, skip_chunk=skip)
    try:
        kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=d["s0"])
        status = kda.device_status()
        detail = kda.lib().kda_last_error().decode()
    finally:
        kda.debug_fault_injection(0, -1)
    assert status == kda.KDA_ERR_TIMEOUT, (status, detail)
    assert "site mask" in detail
    # the status word was cleared by the read; the context is usable and the next call is right
    assert kda.device_status() == kda.KDA_OK
    o, fs = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=d["s0"])
    torch.cuda.synchronize()
    assert kda.device_status() == kda.KDA_OK
    hs = torch.tensor([0, 37, 63])
    sub = {n: (inp[n].index_select(2, hs) if n != "s0" else inp[n].index_select(1, hs))
           for n in ("q", "k", "v", "g", "beta", "s0")}
    eo, es = _oracle_check(sub, o.cpu().index_select(2, hs), fs.cpu().index_select(1, hs))
    assert eo < TOL and es < TOL, (eo, es)
    assert np.isfinite(f64(o)).all()


def test_default_wait_bound_is_restored(kda):
    """After the hook is turned off, a segmented call (map, combine and output
    passes, all with bounded waits) runs without any wait giving up."""
    inp = synth.op_inputs(B=1, H=16, T=3000, s0_std=0.02, seed=42, device="cuda")
    assert kda.chunk_fwd_segments(1, 3000, 16)[0] > 0
    kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], initial_state=inp["s0"])
    assert kda.device_status() == kda.KDA_OK
