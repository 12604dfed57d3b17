#!/usr/bin/env python
"""KDA on B200: prefill tokens/s at B=1, H=16, T=65536 and decode state GB/s.

One step = one ``kda_chunk_fwd`` call over a B=1, H=16, T=65536, d=128 bf16
sequence with a random fp32 initial state (plan; every segment's map with its
chunk products exported; combine; every segment's output).  The decode figure is measured in the same run on the
B=256, H=32 decode workload (512 MiB fp32 state updated in place).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torch.distributed.run, one rank per GPU; every rank runs its
own independent sequence (weak scaling, no collective on the data path) and
the step time is the max over ranks.  ``--impl reference`` times the fp64
oracle (the plain CPU statement of the method) on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

T_PREFILL, H_PREFILL, D = 65536, 16, 128
BYTES_PER_TOKEN_HEAD = 3 * D * 2 + D * 2 + D * 4 + 4   # q,k,v + o (bf16), g (fp32), beta
GDN_BYTES_PER_TOKEN_HEAD = 3 * D * 2 + D * 2 + 4 + 4  # q,k,v + o (bf16), one fp32 gate, beta
FLOP_PER_TOKEN_HEAD = 6 * D * D + 3 * 64 * D + 64 * 64  # the pages' per-head count, C = 64


METRIC = "KDA prefill tokens/s (H=16,T=64K) + decode state GB/s, % of B200 roofline"


def profiled_traffic(summary: str, source: str):
    """DRAM bytes per launch recorded by an ncu capture in profiles/, or None when the
    kernel source has changed since the counters were taken (source hash mismatch)."""
    import hashlib
    try:
        text = open(os.path.join(ROOT, "profiles", summary)).read()
        fields = dict(line.split(":", 1) for line in text.splitlines() if line.startswith(("dram_bytes_per_launch", "kernel_source_sha256")))
        digest = hashlib.sha256(open(os.path.join(ROOT, source), "rb").read()).hexdigest()
        if fields.get("kernel_source_sha256", "").strip() != digest:
            return None
        return float(fields["dram_bytes_per_launch"].strip())
    except Exception:
        return None


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-i", str(self.gpu),
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "samples": len(sm),
                "reasons": sorted(reasons)}


def cpu_oracle_sample(T_s: int, H_s: int, seed: int = 77):
    """Time the fp64 oracle on H_s heads x T_s tokens of the prefill workload."""
    import numpy as np
    import oracle
    import synth
    inp = synth.op_inputs(**{**synth.prefill_sweep(T_PREFILL), "T": T_s, "H": H_s, "seed": seed})
    f = lambda t: t.double().numpy()  # noqa: E731
    args = [f(inp[n]) for n in ("q", "k", "v", "g", "beta")]
    s0 = f(inp["s0"])
    t0 = time.perf_counter()
    oracle.kda_recurrent(*args, s0=s0)
    dt = time.perf_counter() - t0
    return dt, oracle.num_threads()


class Ranks:
    """One process per GPU (or per CPU rank under gloo): rank ids from the launcher's
    environment, a barrier, and the max of a per-rank number over all ranks.  Every rank
    takes the same collective steps in the same order; the process group has a short
    timeout so that ranks waiting for a missing peer end with an error."""

    def __init__(self, backend: str, device=None, timeout_s: int = 120):
        import datetime
        import torch.distributed as dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.device = device
        self._dist = dist
        if self.world > 1:
            kw = {"device_id": device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)

    def barrier(self):
        if self.world > 1:
            self._dist.barrier()

    def max_over_ranks(self, x: float) -> float:
        if self.world == 1:
            return x
        import torch
        t = torch.tensor([x], device=self.device, dtype=torch.float64)
        self._dist.all_reduce(t, op=self._dist.ReduceOp.MAX)
        return float(t.item())

    def seed(self, base: int) -> int:
        """Each rank draws its own independent sequence (weak scaling)."""
        return base + 1000 * self.rank

    def close(self):
        if self.world > 1:
            self._dist.destroy_process_group()


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    T_s, H_s = 2048, H_PREFILL
    times = []
    cores = 1
    for i in range(args.warmup + args.steps):
        dt, cores = cpu_oracle_sample(T_s, H_s, seed=100 + i)
        if i >= args.warmup:
            times.append(dt)
    t = statistics.mean(times)
    value = T_s / t  # tokens/s with all 16 heads of each token
    line = {
        "metric": METRIC, "impl": "reference", "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"KDA prefill B=1 H=16 d=128, oracle sample of {T_s} tokens x {H_s} heads per step",
                   "l2": "n/a (host)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{T_s} tokens x {H_s} heads of the B=1,H=16,T=65536 prefill, per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def time_layer(kda, synth, dev, rank, time_calls, tc_peak, world):
    """The KDA layer: d_model=2048, H=16, rank 128, 65536 packed tokens in 8 sequences, random-init weights."""
    import torch
    lc = synth.LAYER_65K
    lx, lW, lcu = synth.layer_inputs(d_model=lc["d_model"], H=lc["H"], Ttot=lc["Ttot"], nseq=lc["nseq"],
                                     rank=lc["rank"], seed=lc["seed"] + rank, device=dev)
    lpk = kda.pack_layer_weights(lW)
    lcu_d = torch.tensor(lcu, dtype=torch.int32, device=dev)
    ly = torch.empty_like(lx)
    lfs = torch.empty((lc["nseq"], lc["H"], D, D), device=dev, dtype=torch.float32)
    lws = torch.empty(kda.layer_fwd_workspace_bytes(lc["Ttot"], lc["d_model"], lc["H"], lc["rank"], lc["nseq"]),
                      device=dev, dtype=torch.uint8)
    ms = time_calls(lambda: kda.layer_fwd(lx, lpk, lcu_d, out=ly, final_state=lfs, workspace=lws), 5)
    HDl, dm, rk = lc["H"] * D, lc["d_model"], lc["rank"]
    gemm_flop = 2 * lc["Ttot"] * (dm * (3 * HDl + 2 * rk + lc["H"]) + 2 * rk * HDl + HDl * dm)
    flop = gemm_flop + FLOP_PER_TOKEN_HEAD * lc["Ttot"] * lc["H"]
    # the two large projections alone, through kda_linear_bf16 (the layer's GEMM kernel)
    gemms = {}
    for name, n_out, k_in, w in (("input_projection", lpk["W_in"].shape[0], dm, lpk["W_in"]),
                                  ("output_projection", dm, HDl, lpk["W_o"])):
        a = torch.randn((lc["Ttot"], k_in), device=dev, generator=torch.Generator(device=dev).manual_seed(9)
                        ).to(torch.bfloat16)
        yo = torch.empty((lc["Ttot"], (n_out + 7) // 8 * 8), device=dev, dtype=torch.bfloat16)[:, :n_out]
        gms = time_calls(lambda: kda.linear(a, w, out=yo), 10)
        gf = 2 * lc["Ttot"] * n_out * k_in
        gemms[name] = {"M": lc["Ttot"], "N": n_out, "K": k_in, "ms": gms, "tflops": gf / (gms / 1e3) / 1e12,
                       "frac": gf / (gms / 1e3) / 1e12 / tc_peak}
        del a, yo
    return {"workload": "KDA layer d_model=2048 H=16 rank=128, 65536 packed tokens (8 sequences), "
                        "random-init bf16 weights", "ms_per_call": ms,
            "tokens_per_s": world * lc["Ttot"] / (ms / 1e3), "tflops": flop / (ms / 1e3) / 1e12,
            "gemm_tflop_per_call": gemm_flop / 1e12, "tensor_peak_tflops": tc_peak,
            "frac": flop / (ms / 1e3) / 1e12 / tc_peak, "gemm": gemms}


DPLR_BYTES_PER_TOKEN_HEAD = 5 * D * 2 + D * 2 + D * 4 + 4  # q,k,v,a,b + o (bf16), g (fp32), beta


def time_sweep(kda, synth, dev, rank, time_calls, hbm_peak, world, ms_64k, gdn_ms_64k):
    """The pages' length sweep (B=1, H=16, T = 8K..64K) for KDA, its scalar-gate special case
    (gated DeltaNet) and the untied DPLR kernel, each as tokens/s and as the fraction of HBM
    bandwidth its algorithmic bytes reach; plus KDA against DPLR at T=65536 with neither
    kernel running the segment scan (B=4, H=16: 64 CTAs, one per sequence and head)."""
    import torch
    rows = []
    for T in synth.PREFILL_SWEEP_T:
        cfg = dict(synth.prefill_sweep(T))
        cfg["seed"] += 1000 * rank
        row = {"T": T}
        if T == T_PREFILL and ms_64k is not None:
            kms, gms = ms_64k, gdn_ms_64k
        else:
            inp = synth.op_inputs(**cfg, device=dev)
            o, fs = torch.empty_like(inp["q"]), torch.empty_like(inp["s0"])
            ws = torch.empty(kda.chunk_fwd_workspace_bytes(1, T, H_PREFILL), device=dev, dtype=torch.uint8)
            args5 = [inp[n] for n in ("q", "k", "v", "g", "beta")]
            kms = time_calls(lambda: kda.chunk_fwd(*args5, initial_state=inp["s0"], out=o, final_state=fs,
                                                   workspace=ws), 10)
            gs = inp["g"][..., 0].contiguous()
            gms = time_calls(lambda: kda.gdn_chunk_fwd(args5[0], args5[1], args5[2], gs, args5[4],
                                                       initial_state=inp["s0"], out=o, final_state=fs,
                                                       workspace=ws), 10)
            del inp, o, fs, ws, args5, gs
        dp = synth.dplr_inputs(**cfg, device=dev)
        do, dfs = torch.empty_like(dp["q"]), torch.empty_like(dp["s0"])
        dargs = [dp[n] for n in ("q", "k", "v", "a", "b", "g", "beta")]
        dms = time_calls(lambda: kda.dplr_chunk_fwd(*dargs, initial_state=dp["s0"], out=do, final_state=dfs), 3)
        del dp, do, dfs, dargs
        for name, ms, bpt in (("kda", kms, BYTES_PER_TOKEN_HEAD), ("gdn", gms, GDN_BYTES_PER_TOKEN_HEAD),
                              ("dplr", dms, DPLR_BYTES_PER_TOKEN_HEAD)):
            gbs = bpt * T * H_PREFILL / (ms / 1e3) / 1e9
            row[name] = {"ms": ms, "tokens_per_s": world * T / (ms / 1e3), "hbm_frac": gbs / hbm_peak}
        rows.append(row)
    # like for like at the pages' comparison length: 64 (sequence, head) pairs, one CTA each
    B4, T4 = 4, T_PREFILL
    dp = synth.dplr_inputs(B=B4, H=H_PREFILL, T=T4, s0_std=0.02, seed=31 + rank, device=dev)
    do, dfs = torch.empty_like(dp["q"]), torch.empty_like(dp["s0"])
    assert kda.chunk_fwd_segments(B4, T4, H_PREFILL) == (0, 0)
    ws = torch.empty(kda.chunk_fwd_workspace_bytes(B4, T4, H_PREFILL), device=dev, dtype=torch.uint8)
    kms = time_calls(lambda: kda.chunk_fwd(*(dp[n] for n in ("q", "k", "v", "g", "beta")), initial_state=dp["s0"],
                                           out=do, final_state=dfs, workspace=ws), 3)
    dms = time_calls(lambda: kda.dplr_chunk_fwd(*(dp[n] for n in ("q", "k", "v", "a", "b", "g", "beta")),
                                                initial_state=dp["s0"], out=do, final_state=dfs), 3)
    del dp, do, dfs, ws
    return {"workload": "B=1 H=16 d=128, T = 8K..64K (prefill distributions); kda = per-channel gates, "
                        "gdn = one gate per token-head, dplr = untied a, b",
            "lengths": rows,
            "no_scan_64k": {"workload": f"B={B4} H=16 T={T4}: 64 CTAs, one per (sequence, head); neither "
                                        "kernel segments", "kda_ms": kms, "dplr_ms": dms,
                            "dplr_over_kda": dms / kms}}


def run_ours(args):
    import torch

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    world, rank = ranks.world, ranks.rank

    import gated_delta_rule_123_b200 as kda
    import synth

    barrier, max_over_ranks = ranks.barrier, ranks.max_over_ranks

    hbm_peak, tc_peak, peak_kind = measured_peaks()
    T = args.T
    cfg = dict(synth.prefill_sweep(T))
    cfg["seed"] = ranks.seed(cfg["seed"])
    inp = synth.op_inputs(**cfg, device=dev)
    q, k, v, g, beta, s0 = (inp[n] for n in ("q", "k", "v", "g", "beta", "s0"))
    o = torch.empty_like(q)
    fs = torch.empty_like(s0)
    wsz = kda.chunk_fwd_workspace_bytes(1, T, H_PREFILL)
    ws = torch.empty(wsz, device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)

    def step():
        kda.chunk_fwd(q, k, v, g, beta, initial_state=s0, out=o, final_state=fs, workspace=ws)

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def time_calls(fn, n):
        for _ in range(2):
            fn()
        barrier()
        torch.cuda.synchronize()
        start.record(stream)
        for _ in range(n):
            fn()
        end.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(start.elapsed_time(end) / n)

    if args.gemm_only:  # the layer's input projection shape with args.gemm_m rows (profiling runs)
        lc = synth.LAYER_65K
        n_out = 3 * lc["H"] * D + 2 * lc["rank"] + lc["H"]
        gen = torch.Generator(device=dev).manual_seed(9)
        a = torch.randn((args.gemm_m, lc["d_model"]), device=dev, generator=gen).to(torch.bfloat16)
        w = (0.02 * torch.randn((n_out, lc["d_model"]), device=dev, generator=gen)).to(torch.bfloat16)
        yo = torch.empty((args.gemm_m, n_out), device=dev, dtype=torch.bfloat16)
        gms = time_calls(lambda: kda.linear(a, w, out=yo), args.steps)
        tf = 2 * args.gemm_m * n_out * lc["d_model"] / (gms / 1e3) / 1e12
        if rank == 0:
            print(json.dumps({"metric": "GEMM TFLOP/s", "value": tf, "unit": "TFLOP/s", "ms": gms,
                              "config": {"workload": f"y = x W^T, M={args.gemm_m} N={n_out} K={lc['d_model']} bf16"},
                              "frac": tf / tc_peak}), flush=True)
        ranks.close()
        return 0
    if args.dplr_only:  # the untied DPLR kernel at B=1, H=16, T=args.T (profiling runs)
        dp = synth.dplr_inputs(**synth.prefill_sweep(T), device=dev)
        do, dfs = torch.empty_like(dp["q"]), torch.empty_like(dp["s0"])
        dms = time_calls(lambda: kda.dplr_chunk_fwd(*(dp[n] for n in ("q", "k", "v", "a", "b", "g", "beta")),
                                                    initial_state=dp["s0"], out=do, final_state=dfs), args.steps)
        if rank == 0:
            print(json.dumps({"metric": "DPLR prefill tokens/s", "value": T / (dms / 1e3), "unit": "tokens/s",
                              "ms": dms, "config": {"workload": f"untied DPLR B=1 H=16 T={T}"}}), flush=True)
        ranks.close()
        return 0
    if args.layer_only:
        layer = time_layer(kda, synth, dev, rank, time_calls, tc_peak, world)
        if rank == 0:
            print(json.dumps({"metric": "KDA layer tokens/s", "value": layer["tokens_per_s"], "unit": "tokens/s",
                              "config": {"workload": layer["workload"]}, "layer": layer}), flush=True)
        ranks.close()
        return 0

    sampler = ClockSampler(local)
    sampler.start()
    t_w = time.perf_counter()
    n_w = 0
    while n_w < args.warmup or time.perf_counter() - t_w < args.warmup_seconds:
        step()
        n_w += 1
        if n_w % 10 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    assert kda.device_status() == 0

    def timed_steps(fn, traces):
        """Time args.steps calls of fn.  The calls are captured into one CUDA graph and
        replayed, so host-side jitter between calls cannot leave the GPU idle.  The
        per-launch breakdown comes from a second graph of the same calls with the
        library's trace events (event nodes between the launches), replayed after the
        timed one, so that the timed graph holds the calls alone.  --eager times the
        traced calls as issued."""
        for tr in traces:  # create the events outside the capture
            for e in tr:
                e.record(stream)
        graph, traced, timing = None, None, "eager: K calls issued back to back"
        if not args.eager:
            try:
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph):
                    for i in range(args.steps):
                        fn()
                traced = torch.cuda.CUDAGraph()
                with torch.cuda.graph(traced):
                    for i in range(args.steps):
                        kda.set_trace_events(traces[i])
                        fn()
                kda.set_trace_events(None)
                graph.replay()  # untimed: uploads the graphs
                traced.replay()
                torch.cuda.synchronize()
                timing = ("one CUDA graph of the K calls, replayed once; the per-launch times come from a "
                          "second graph with trace events between the launches")
            except Exception as exc:  # fall back to timing the calls as issued
                kda.set_trace_events(None)
                graph = traced = None
                torch.cuda.synchronize()
                print(f"bench: CUDA graph capture failed ({exc}); timing eagerly", file=sys.stderr)
        assert kda.device_status() == 0
        barrier()
        torch.cuda.synchronize()
        start.record(stream)
        if graph is not None:
            graph.replay()
        else:
            for i in range(args.steps):
                kda.set_trace_events(traces[i])
                fn()
        end.record(stream)
        torch.cuda.synchronize()
        barrier()
        kda.set_trace_events(None)
        if traced is not None:  # untimed: the per-launch breakdown
            traced.replay()
            torch.cuda.synchronize()
        return start.elapsed_time(end) / args.steps, timing

    # timed region: K steps
    traces = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    ms, timing = timed_steps(step, traces)
    clocks = sampler.stop()
    ms = max_over_ranks(ms)
    out_ms = statistics.mean(tr[3].elapsed_time(tr[4]) for tr in traces)
    sum_ms = statistics.mean(tr[1].elapsed_time(tr[2]) for tr in traces)
    comb_ms = statistics.mean(tr[2].elapsed_time(tr[3]) for tr in traces)
    plan_ms = statistics.mean(tr[0].elapsed_time(tr[1]) for tr in traces)
    assert kda.device_status() == 0
    value = world * T / (ms / 1e3)

    # Roofline per launch, algorithmic bytes of the tokens each processes: phase 1 runs every
    # segment's map (q, k, v, g, beta read, no output: 1284 B per token-head); phase 2 writes
    # every token's output (1540 B).  Unsegmented calls run one launch, timed as phase 2.  The
    # longer launch is reported as dominant.
    seg0, mid = kda.chunk_fwd_segments(1, T, H_PREFILL)
    p1_bytes = 0 if seg0 == 0 else (BYTES_PER_TOKEN_HEAD - 2 * D) * T * H_PREFILL
    p2_bytes = BYTES_PER_TOKEN_HEAD * T * H_PREFILL
    launches = {"phase1_segment_maps": {"ms": sum_ms, "algorithmic_bytes": p1_bytes},
                "phase2_segment_outputs": {"ms": out_ms, "algorithmic_bytes": p2_bytes}}
    for rec in launches.values():
        rec["achieved_gbs"] = rec["algorithmic_bytes"] / (rec["ms"] / 1e3) / 1e9 if rec["ms"] > 0 else 0.0
        rec["frac"] = rec["achieved_gbs"] / hbm_peak
    dom = max(launches, key=lambda n: launches[n]["ms"])
    traffic = profiled_traffic("chunk_phase1_T65536_traffic.md", "gated_delta_rule_123_b200/csrc/kda_chunk.cu")
    roofline = {"bound": "hbm", "achieved": launches[dom]["achieved_gbs"], "peak": hbm_peak, "unit": "GB/s",
                "frac": launches[dom]["frac"],
                "traffic": traffic if (T == T_PREFILL and dom.startswith("phase1")) else None,
                "traffic_unit": "bytes per launch", "algorithmic_bytes": launches[dom]["algorithmic_bytes"],
                "kernel": dom, "launches": launches, "segment_tokens": {"first": seg0, "following": mid},
                "peak_kind": peak_kind,
                "step_frac": BYTES_PER_TOKEN_HEAD * T * H_PREFILL / (ms / 1e3) / 1e9 / hbm_peak,
                "kernel_ms": {"plan": plan_ms, "segment_maps": sum_ms, "combine": comb_ms,
                              "segment_outputs": out_ms},
                "tensor_tflops_step": FLOP_PER_TOKEN_HEAD * T * H_PREFILL / (ms / 1e3) / 1e12,
                "tensor_peak": tc_peak}

    if args.prefill_only:
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": value, "unit": "tokens/s", "ms_per_step": ms,
                              "config": {"workload": f"KDA prefill B=1 H=16 T={T} (prefill only)", "timing": timing},
                              "roofline": roofline}), flush=True)
        ranks.close()
        return 0

    # decode: B=256, H=32, state updated in place (inputs cycled from a pool of 8 seeded steps)
    dcfg = synth.DECODE_B256
    B, H = dcfg["B"], dcfg["H"]
    S = synth.decode_state(B, H, seed=dcfg["seed"] + rank, device=dev)
    pool = [synth.decode_step_inputs(B, H, i, seed=dcfg["seed"], device=dev) for i in range(8)]
    od = torch.empty_like(pool[0]["q"])

    def dstep(i):
        p = pool[i % 8]
        kda.decode_step(p["q"], p["k"], p["v"], p["g"], p["beta"], S, out=od)

    for i in range(5):
        dstep(i)
    n_dec = 200
    barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(n_dec):
        dstep(i)
    end.record(stream)
    torch.cuda.synchronize()
    dec_us = max_over_ranks(start.elapsed_time(end) / n_dec * 1e3)
    dec_bytes = 2 * B * H * D * D * 4 + B * H * (4 * D * 2 + D * 4 + 4)
    dec_gbs = dec_bytes / (dec_us / 1e6) / 1e9
    assert kda.device_status() == 0

    # fused recurrent segments: 16 tokens per sequence on the decode shape, state in place
    rT = 16
    rin = synth.op_inputs(B=B, H=H, T=rT, seed=dcfg["seed"] + 7 + rank, device=dev)
    orr = torch.empty_like(rin["q"])

    def rstep():
        kda.recurrent_fwd(rin["q"], rin["k"], rin["v"], rin["g"], rin["beta"], S, out=orr)

    for _ in range(3):
        rstep()
    n_rec = 50
    barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(n_rec):
        rstep()
    end.record(stream)
    torch.cuda.synchronize()
    rec_us = max_over_ranks(start.elapsed_time(end) / n_rec * 1e3)
    assert kda.device_status() == 0

    # gated DeltaNet fast path on the same workload: one log-gate per (token, head)
    gs = g[..., 0].contiguous()

    def gstep():
        kda.gdn_chunk_fwd(q, k, v, gs, beta, initial_state=s0, out=o, final_state=fs, workspace=ws)

    for _ in range(3):
        gstep()
    barrier()
    torch.cuda.synchronize()
    gtr = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    gdn_ms, _ = timed_steps(gstep, gtr)
    gdn_ms = max_over_ranks(gdn_ms)
    gdn_kernel_ms = {name: statistics.mean(tr[a].elapsed_time(tr[a + 1]) for tr in gtr)
                     for a, name in enumerate(("plan", "segment_maps", "combine", "segment_outputs"))}
    assert kda.device_status() == 0
    gdn_bytes = GDN_BYTES_PER_TOKEN_HEAD * T * H_PREFILL

    # untied DPLR comparison kernel: at the pages' comparison shape (B=1, H=16, T; one CTA per head,
    # no segment scan) and, against KDA, at a shape where neither kernel segments (B=16, H=16, T=4096)

    dp = synth.dplr_inputs(B=1, H=H_PREFILL, T=T, s0_std=0.02, seed=cfg["seed"] + 11, device=dev)
    dargs = [dp[n] for n in ("q", "k", "v", "a", "b", "g", "beta")]
    dplr_ms = time_calls(lambda: kda.dplr_chunk_fwd(*dargs, initial_state=dp["s0"], out=o, final_state=fs), 3)
    del dp, dargs
    eq = synth.dplr_inputs(B=16, H=H_PREFILL, T=4096, s0_std=0.02, seed=cfg["seed"] + 12, device=dev)
    eo_, efs = torch.empty_like(eq["q"]), torch.empty_like(eq["s0"])
    eq_dplr_ms = time_calls(lambda: kda.dplr_chunk_fwd(*(eq[n] for n in ("q", "k", "v", "a", "b", "g", "beta")),
                                                       initial_state=eq["s0"], out=eo_, final_state=efs), 5)
    eq_kda_ms = time_calls(lambda: kda.chunk_fwd(*(eq[n] for n in ("q", "k", "v", "g", "beta")),
                                                 initial_state=eq["s0"], out=eo_, final_state=efs), 5)
    del eq, eo_, efs
    assert kda.device_status() == 0

    # backward (recurrent reverse mode) on B=1 H=16 T=8192, all six gradients
    bT = 8192
    bw = synth.op_inputs(B=1, H=H_PREFILL, T=bT, s0_std=0.02, seed=cfg["seed"] + 13, device=dev)
    bdo = torch.randn(bw["q"].shape, device=dev, generator=torch.Generator(device=dev).manual_seed(7)).to(bw["q"].dtype)
    bws = torch.empty(kda.lib().kda_recurrent_bwd_workspace(1, bT, H_PREFILL), device=dev, dtype=torch.uint8)
    bwd_ms = time_calls(lambda: kda.recurrent_bwd(bw["q"], bw["k"], bw["v"], bw["g"], bw["beta"], bdo,
                                                  initial_state=bw["s0"], workspace=bws), 2)
    del bw, bdo, bws
    assert kda.device_status() == 0

    layer = time_layer(kda, synth, dev, rank, time_calls, tc_peak, world)
    assert kda.device_status() == 0
    sweep = time_sweep(kda, synth, dev, rank, time_calls, hbm_peak, world, ms if T == T_PREFILL else None,
                       gdn_ms if T == T_PREFILL else None)
    assert kda.device_status() == 0

    # End to end through the public call with host buffers (pinned), copies inside the timed
    # region.  Steps are pipelined as a serving loop would run them: step i+1's inputs go
    # host -> device on their own stream while step i computes and its result comes back on a
    # third stream (two device buffer sets, events order the reuse).  Every step still copies
    # its own inputs in and reads its own result out.
    hq, hk, hv, hg, hb, hs0 = (t.cpu().pin_memory() for t in (q, k, v, g, beta, s0))
    host_in = (hq, hk, hv, hg, hb, hs0)
    host_out = [(torch.empty(o.shape, dtype=o.dtype, pin_memory=True),
                 torch.empty(fs.shape, dtype=fs.dtype, pin_memory=True)) for _ in range(2)]
    dev_in = [[torch.empty_like(t) for t in (q, k, v, g, beta, s0)] for _ in range(2)]
    dev_out = [(torch.empty_like(o), torch.empty_like(fs)) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = host_out[0][0].numel() * host_out[0][0].element_size() + host_out[0][1].numel() * host_out[0][1].element_size()
    e2e_steps = max(2, min(args.steps, 8))
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(n):
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        for i in range(n):
            b = i & 1
            if i >= 2:
                s_in.wait_event(ev_comp[b])  # step i-2 has consumed input set b
            with torch.cuda.stream(s_in):
                for d_, h_ in zip(dev_in[b], host_in):
                    d_.copy_(h_, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])  # step i-2's result has been read out of set b
            dq, dk, dv, dg, db, ds0 = dev_in[b]
            kda.chunk_fwd(dq, dk, dv, dg, db, initial_state=ds0, out=dev_out[b][0], final_state=dev_out[b][1],
                          workspace=ws)
            ev_comp[b].record(stream)
            s_out.wait_event(ev_comp[b])
            with torch.cuda.stream(s_out):
                host_out[b][0].copy_(dev_out[b][0], non_blocking=True)
                host_out[b][1].copy_(dev_out[b][1], non_blocking=True)
                ev_out[b].record(s_out)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    o_ref = kda.chunk_fwd(q, k, v, g, beta, initial_state=s0, workspace=ws)[0].cpu()
    e2e_run(2)
    torch.cuda.synchronize()
    barrier()
    start.record(stream)
    e2e_run(e2e_steps)
    end.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(start.elapsed_time(end) / e2e_steps)
    assert torch.equal(host_out[(e2e_steps - 1) & 1][0], o_ref)  # the last step's result came back

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        T_s, H_s = args.T, H_PREFILL  # the whole prefill workload, one step
        dt, cores = cpu_oracle_sample(T_s, H_s)
        cpu = {"value": T_s / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{T_s} tokens x {H_s} heads of the B=1,H=16,T=65536 prefill ({dt:.1f} s)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"KDA prefill B=1 H=16 T={T} d=128 bf16, fp32 g/beta/state "
                                   "(one independent sequence per GPU)",
                       "l2": "inputs larger than L2 (1.6 GB per step)", "parallelism": f"replicas x{world}",
                       "timing": timing},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": {"value": world * T / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": 4 * args.steps,
            "clocks": clocks,
            "decode": {"workload": "B=256 H=32 d=128, fp32 state in place", "us_per_step": dec_us,
                       "gbs": dec_gbs, "peak_gbs": hbm_peak, "frac": dec_gbs / hbm_peak,
                       "tokens_per_s": world * B / (dec_us / 1e6)},
            "recurrent": {"workload": f"B={B} H={H} segments of {rT} tokens, fp32 state in place",
                          "us_per_call": rec_us, "tokens_per_s": world * B * rT / (rec_us / 1e6),
                          "us_per_token": rec_us / rT},
            "dplr": {"workload": f"untied DPLR prefill B=1 H=16 T={T} (one CTA per head, no segment scan)",
                     "ms_per_step": dplr_ms, "tokens_per_s": world * T / (dplr_ms / 1e3),
                     "equal_parallelism": {"workload": "B=16 H=16 T=4096, neither kernel segments",
                                           "dplr_ms": eq_dplr_ms, "kda_ms": eq_kda_ms,
                                           "dplr_over_kda": eq_dplr_ms / eq_kda_ms}},
            "backward": {"workload": "B=1 H=16 T=8192: dq, dk, dv, dg, dbeta, dS0 by recurrent reverse mode",
                         "ms_per_call": bwd_ms, "tokens_per_s": world * bT / (bwd_ms / 1e3)},
            "layer": layer,
            "sweep": sweep,
            "gdn": {"workload": f"gated DeltaNet prefill B=1 H=16 T={T}, one fp32 log-gate per token-head",
                    "ms_per_step": gdn_ms, "tokens_per_s": world * T / (gdn_ms / 1e3),
                    "step_gbs": gdn_bytes / (gdn_ms / 1e3) / 1e9,
                    "step_frac": gdn_bytes / (gdn_ms / 1e3) / 1e9 / hbm_peak, "kernel_ms": gdn_kernel_ms},
        }
        print(json.dumps(line), flush=True)
    ranks.close()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--T", type=int, default=T_PREFILL, help="prefill length (profiling runs use a smaller one)")
    ap.add_argument("--prefill-only", action="store_true", help="skip decode, e2e and the CPU baseline")
    ap.add_argument("--eager", action="store_true", help="time the prefill calls as issued, not as one CUDA graph")
    ap.add_argument("--layer-only", action="store_true", help="time only the KDA layer (profiling runs)")
    ap.add_argument("--gemm-only", action="store_true", help="time only the layer's input-projection GEMM")
    ap.add_argument("--gemm-m", type=int, default=65536, help="rows of the --gemm-only GEMM")
    ap.add_argument("--dplr-only", action="store_true", help="time only the untied DPLR kernel at --T")
    ap.add_argument("--warmup-seconds", type=float, default=1.5, help="minimum warm-up time (clock sampling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
