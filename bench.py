#!/usr/bin/env python
"""Benchmark of paged absorbed-MLA decode (plan + split scan + combine) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--only]
                    [--no-side] [--tokens T] [--impl ours|reference]

One step = one pass of the whole hot path over one batch: the split planner, the
split scan (the dominant kernel) and the LSE combine, on inputs already resident in HBM.
Prints ONE JSON line on rank 0.  Its headline workload is long_m256 (B=16, s_q=16,
H=16, 131,072 cached tokens per request: the largest single-GPU configuration); value =
KV-read GB/s of the whole job (bytes of cache rows the decode must read, summed over
ranks, divided by the slowest rank's device time); us_per_call is the per-step latency.
The L2 (126 MB) is flushed between timed steps, outside the timed events, by a 256 MB
write followed by a 256 MB read of another buffer (the read writes the flush's dirty
lines back before the timed kernels start).  The same run then measures every other workload (tiny, agent_spec,
ragged_rownorm, fp8_batch) the same way; each has its own record under "workloads",
with its roofline fraction and its own clock record (--only skips them).

Beside the step the line carries, each timed on its own with CUDA events and the L2
flushed before every call: the paged KV append of the drafts' rows (kv_append), the
projections either side of the latent attention (absorb_project), both per workload,
and a long-prefix chunked prefill on the same path (prefill: one request, 1024 query
tokens x 16 heads at the end of a 65,536-token cache).  --tokens T gives every request
T tokens: a reduced case for profiler captures, never a bench number.

Multi-GPU (torchrun): every rank decodes its own replica of the workload (requests are
independent; there is no data-path collective), time = max over ranks, scaling weak.

--impl reference times the float64 CPU oracle on a bounded sample of the same workload
and reports it in the same metric, extrapolated by rows (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from mla_attention_decode_paged_b200 import workloads as W  # noqa: E402

DEFAULT_WORKLOAD = "long_m256"  # the largest single-GPU configuration: B=16, s_q=16, H=16, 131,072 tokens each
METRIC = "MLA decode \u00b5s/call and KV-read GB/s (% of B200 HBM/tensor roofline)"  # value in GB/s; us_per_call beside it
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}  # B200 datasheet (dense bf16), for context
KERNEL_SOURCES = ["mla_attention_decode_paged_b200/csrc/mla_decode_sm100.cu",
                  "mla_attention_decode_paged_b200/csrc/mla_decode_sm100_e4m3.cu",
                  "mla_attention_decode_paged_b200/csrc/mla_scan_common.cuh",
                  "mla_attention_decode_paged_b200/csrc/mla_common.cuh",
                  "mla_attention_decode_paged_b200/csrc/sm100_ptx.cuh"]


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload):
    """DRAM bytes per launch of the scan kernel from the committed ncu summary, if it was
    taken on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("kernel_hash") != kernel_hash():
        return None
    return e.get("dram_bytes_per_launch")


def workload_desc(wl):
    s = wl.spec
    lens = wl.seq_lens
    return (f"{s.name}: B={s.B} s_q={s.s_q} H={s.H} (M={s.M}) T={int(lens.min())}..{int(lens.max())} "
            f"(sum {int(lens.sum())}) page=64 {'e4m3' if s.kv_dtype else 'bf16'} KV, "
            f"{'causal' if s.causal else 'non-causal'}, shuffled block_table, seed {s.seed}")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while alive."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.dev)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def oracle_sample(wl, n_req=None):
    """Time the oracle on n_req requests x a head subset (16-row blocks, enough of them to
    give every host core one); returns (seconds for the full workload, extrapolated by rows and
    by the sampled requests' share of cache tokens, threads used, description)."""
    import oracle
    reqs = list(range(wl.B if n_req is None else max(1, min(wl.B, n_req))))
    # enough 16-row blocks per request that every host core has one (the oracle runs one
    # OpenMP task per request and 16-row block)
    blocks = max(1, -(-len(os.sched_getaffinity(0)) // len(reqs)))
    heads = list(range(max(1, min(wl.H, 16 * blocks // wl.s_q))))
    rows_s = wl.s_q * len(heads)
    t0 = time.perf_counter()
    oracle.mla_decode(wl.q[reqs][:, :, heads], wl.kv, wl.kv_dtype, wl.kv_scale, wl.block_table[reqs],
                      wl.seq_lens[reqs], wl.scale, wl.causal)
    dt = time.perf_counter() - t0
    tok_share = float(wl.seq_lens[reqs].astype(np.int64).sum()) / float(wl.seq_lens.astype(np.int64).sum())
    full = dt * (wl.spec.M / rows_s) / tok_share
    cores = min(len(reqs) * ((rows_s + 15) // 16), len(os.sched_getaffinity(0)))
    desc = (f"oracle on {len(reqs)} of {wl.B} requests x {len(heads)} head(s) x {wl.s_q} drafts = {rows_s} of "
            f"{wl.spec.M} rows per request ({dt:.2f} s), scaled by rows and cache tokens to the full workload")
    return full, cores, desc


def oracle_baseline(wl, target_s=10.0, cap_s=30.0):
    """The oracle timed on about target_s seconds of CPU work (never past cap_s): a pilot
    sample sizes the number of requests, then the sample is repeated until target_s is
    reached.  Returns (seconds for the full workload, threads used, description)."""
    t0 = time.perf_counter()
    pilot, _, _ = oracle_sample(wl, 1)
    pilot_s = time.perf_counter() - t0
    # the pilot ran one request's 16-row sample; a run over n requests costs about n times it
    per_req = max(pilot_s, 1e-3)
    n_req = int(max(1, min(wl.B, target_s / per_req)))
    runs, total, full = 0, 0.0, []
    cores, desc = 0, ""
    while True:
        t1 = time.perf_counter()
        f, cores, desc = oracle_sample(wl, n_req)
        total += time.perf_counter() - t1
        full.append(f)
        runs += 1
        if total >= target_s or total + total / runs > cap_s:
            break
    return (sum(full) / len(full), cores,
            f"{desc}; {runs} run(s), {total:.1f} s of CPU time in all, after a one-request pilot")


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = W.make_workload(args.workload)
    kvb = wl.kv_bytes()
    # size the per-step sample so that the whole run stays within about two minutes
    n_req = wl.B
    t0 = time.perf_counter()
    oracle_sample(wl, n_req)
    first = time.perf_counter() - t0
    n_steps = args.warmup - 1 + args.steps
    if first * n_steps > 120.0:
        n_req = max(1, int(wl.B * 120.0 / (first * n_steps)))
    for _ in range(args.warmup - 1):
        oracle_sample(wl, n_req)
    times = []
    cores, desc = 0, ""
    for _ in range(args.steps):
        t, cores, desc = oracle_sample(wl, n_req)
        times.append(t)
    step = sum(times) / len(times)
    value = kvb / step / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3, "us_per_call": step * 1e6,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(wl), "global_batch": wl.B, "seq_len": int(wl.seq_lens.max()),
                       "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def max_over_ranks(values, world, device):
    """Per-rank totals reduced with MAX over the ranks: the slowest rank sets the job's
    time.  Every rank calls it at the same points, in the same order."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def job_gbs(bytes_per_rank_step, world, steps, total_ms):
    """Whole-job throughput: every rank's bytes over the slowest rank's device time."""
    return bytes_per_rank_step * world * steps / (total_ms * 1e-3) / 1e9


def prefill_measure(args, dev, stream, flush_l2, time_op, B=1, chunk=1024, H=16, T=65536):
    """Long-prefix chunked prefill (mla_prefill) on one request: a chunk of 1024 query
    tokens x 16 heads whose rows end a 65,536-token cache, causal within the chunk.
    FLOPs count every visible (row, token) pair: 2 H (C (T - C) + C (C + 1) / 2) (576 + 512)."""
    import torch
    import mla_attention_decode_paged_b200 as mla
    wl = W.make_workload("agent_spec", B=B, s_q=chunk, H=H, seq_lens=[T] * B, seed=21)
    q = torch.from_numpy(wl.q.view(np.int16)).view(torch.bfloat16).to(dev)
    kv = torch.from_numpy(wl.kv.view(np.int16)).view(torch.bfloat16).to(dev)
    bt = torch.from_numpy(wl.block_table).to(dev)
    sl = torch.from_numpy(wl.seq_lens).to(dev)
    ws = mla.alloc_prefill_workspace(B, chunk, H, int(bt.shape[1]), device=dev)
    out = torch.empty((B, chunk, H, W.DV), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, chunk, H), dtype=torch.float32, device=dev)
    us = time_op(lambda: mla.prefill(q, kv, bt, sl, wl.scale, ws, out, lse, stream=stream))
    if mla.device_status(ws, stream=stream) != 0:
        raise RuntimeError("prefill: device status set")
    pairs = B * H * (chunk * (T - chunk) + chunk * (chunk + 1) // 2)
    flops = 2 * pairs * (W.DQK + W.DV)
    peaks, peak_src = load_peaks()
    tf = flops / (us * 1e-6) / 1e12
    d = mla.mla_prefill_sub_chunk(chunk, H)
    return {"workload": f"B={B} chunk={chunk} H={H} T={T} (prefix {T - chunk} + chunk) bf16 cache, causal in the "
                        f"chunk, seed 21",
            "us_per_call": us, "tflops": tf, "algorithmic_flops": flops, "peak_tflops": peaks["bf16_tflops"],
            "frac_of_bf16_peak": tf / peaks["bf16_tflops"], "peak_source": peak_src, "sub_chunk": d,
            "sub_chunk_requests": B * chunk // d, "kv_bytes": wl.kv_bytes(),
            "note": "runs on the decode path (expand + plan + split scan + combine, 4 launches); L2 flushed before "
                    "each call; the request's 74 MB of cache rows stay in L2 across its sub-chunks"}


def soak(step, flush_l2, dev, seconds):
    import torch
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        for k in range(10):
            flush_l2(k)
            step()
        torch.cuda.synchronize(dev)


def roofline_of(wl, scan_avg_s, traffic):
    """Roofline of the split scan for one launch: HBM-bound (cache bytes) or tensor-bound
    (2 M T 1088 FLOPs) by the workload's intensity against the measured ridge."""
    peaks, peak_src = load_peaks()
    kvb, flops = wl.kv_bytes(), wl.flops()
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if flops / kvb < ridge:
        roof = {"bound": "hbm", "achieved": kvb / scan_avg_s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": flops / scan_avg_s / 1e12, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = traffic
    roof["peak_source"] = f"{peak_src} ({'MEASURED_PEAKS.json' if peak_src == 'measured' else 'profiling recipe'})"
    roof["kernel"] = "mla decode split scan"
    roof["algorithmic_bytes_per_launch"] = kvb
    roof["algorithmic_flops_per_launch"] = flops
    if roof["bound"] == "tensor" and wl.kv_dtype != W.KV_BF16:
        # the e4m3 scan's MMAs take q and P as two e4m3 terms each (bf16 precision), so each
        # product runs twice on the fp8 pipe: its executed FLOPs against the fp8 peak (twice
        # the bf16 one) give the same fraction as these FLOPs against the bf16 peak
        roof["note"] = "bf16-precision FLOPs against the bf16 peak; e4m3 MMAs run each product as two terms"
    nom_peak = NOMINAL_PEAKS["hbm_gbs"] if roof["bound"] == "hbm" else NOMINAL_PEAKS["bf16_tflops"]
    nominal = {"peak": nom_peak, "unit": roof["unit"], "frac": roof["achieved"] / nom_peak,
               "note": "B200 datasheet peak, context only"}
    t_roof = max(kvb / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops"] * 1e12))
    return roof, nominal, t_roof


def measure_workload(name, args, dev, stream, flush_l2, world, headline):
    """One workload: the decode step (plan + split scan + combine) timed with CUDA events,
    the per-kernel pass, clocks sampled during both; for the headline also the CUDA-graph
    replay and the warm-L2 step; end to end through the public calls with host buffers;
    and the side paths (KV append, the projections) on the workload's shapes."""
    import torch
    import mla_attention_decode_paged_b200 as mla

    kw = {} if args.tokens is None else {"seq": ("fixed", args.tokens)}
    wl = W.make_workload(name, **kw)
    q, kv, bt, sl = (torch.from_numpy(wl.q.view(np.int16)).view(torch.bfloat16).to(dev),
                     (torch.from_numpy(wl.kv.view(np.int16)).view(torch.bfloat16) if wl.kv_dtype == W.KV_BF16
                      else torch.from_numpy(wl.kv)).to(dev),
                     torch.from_numpy(wl.block_table).to(dev), torch.from_numpy(wl.seq_lens).to(dev))
    ws = mla.alloc_workspace(wl.B, wl.s_q, wl.H, device=dev)
    out = torch.empty((wl.B, wl.s_q, wl.H, W.DV), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((wl.B, wl.s_q, wl.H), dtype=torch.float32, device=dev)

    def step(ev=None):
        # the three kernels back to back, so that each starts its prologue under the tail
        # of the one before (programmatic dependent launch); events only around the step
        if ev is not None:
            ev[0].record(stream)
        mla.plan(sl, wl.s_q, wl.H, ws, stream=stream)
        mla.decode(q, kv, bt, sl, wl.scale, wl.causal, ws, out, lse, kv_scale=wl.kv_scale, stream=stream)
        if ev is not None:
            ev[1].record(stream)

    def step_split(ev):
        # the same kernels with an event between each pair: per-kernel durations (the events
        # serialise the launches, so this pass is a little slower than the step above)
        ev[0].record(stream)
        mla.plan(sl, wl.s_q, wl.H, ws, stream=stream)
        ev[1].record(stream)
        mla.decode(q, kv, bt, sl, wl.scale, wl.causal, ws, out, lse, kv_scale=wl.kv_scale, stream=stream,
                   scan_only=True)
        ev[2].record(stream)
        mla.combine(ws, wl.B, wl.s_q, wl.H, out, lse, stream=stream)
        ev[3].record(stream)

    for _ in range(args.warmup):
        flush_l2(0)
        step()
    torch.cuda.synchronize(dev)
    assert mla.device_status(ws, stream=stream) == 0
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    evs_split = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    with ClockSampler(dev.index) as clk:
        # The timed steps are short next to the sampler's 200 ms period, so identical
        # untimed steps run for a soak window before and after them; the clock record
        # covers the soak and the timed steps together.
        soak(step, flush_l2, dev, args.soak_s)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        for k in range(args.steps):
            flush_l2(k)  # outside the timed events
            step(evs[k])
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        for k in range(args.steps):
            flush_l2(k)
            step_split(evs_split[k])
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        soak(step, flush_l2, dev, args.soak_s)
    assert mla.device_status(ws, stream=stream) == 0
    step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    plan_ms = [e[0].elapsed_time(e[1]) for e in evs_split]
    scan_ms = [e[1].elapsed_time(e[2]) for e in evs_split]
    comb_ms = [e[2].elapsed_time(e[3]) for e in evs_split]
    tot_ms, tot_scan_ms = max_over_ranks([sum(step_ms), sum(scan_ms)], world, dev)
    kvb, flops = wl.kv_bytes(), wl.flops()
    roof, roof_nominal, t_roof = roofline_of(wl, tot_scan_ms * 1e-3 / args.steps,
                                             ncu_traffic(name) if args.tokens is None else None)
    rec = {"workload": workload_desc(wl), "value": job_gbs(kvb, world, args.steps, tot_ms), "unit": "GB/s",
           "us_per_call": tot_ms / args.steps * 1e3,
           "tflops": flops * world * args.steps / (tot_ms * 1e-3) / 1e12,
           "step_us_p10_p50_p90": [float(np.percentile(step_ms, p)) * 1e3 for p in (10, 50, 90)],
           "breakdown_us": {"plan": statistics.median(plan_ms) * 1e3, "scan": statistics.median(scan_ms) * 1e3,
                            "combine": statistics.median(comb_ms) * 1e3,
                            "note": "a second pass of K steps with events between the kernels"},
           "roofline_us": t_roof * 1e6, "frac_of_roofline_step": t_roof / (tot_ms * 1e-3 / args.steps),
           "roofline": roof, "roofline_nominal": roof_nominal, "clocks": clk.summary(),
           "kv_bytes": kvb, "flops": flops}

    if headline:
        # the same step replayed from a CUDA graph (captured once; launch overhead removed)
        try:
            g = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream(dev)
            cap.wait_stream(stream)
            with torch.cuda.graph(g, stream=cap):
                mla.plan(sl, wl.s_q, wl.H, ws, stream=cap)
                mla.decode(q, kv, bt, sl, wl.scale, wl.causal, ws, out, lse, kv_scale=wl.kv_scale, stream=cap)
            torch.cuda.synchronize(dev)
            gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
            for k in range(args.warmup):
                flush_l2(k)
                g.replay()
            torch.cuda.synchronize(dev)
            for k in range(args.steps):
                flush_l2(k)
                gev[k][0].record(stream)
                g.replay()
                gev[k][1].record(stream)
            torch.cuda.synchronize(dev)
            assert mla.device_status(ws, stream=stream) == 0
            gms = sorted(e[0].elapsed_time(e[1]) for e in gev)
            (g_ms,) = max_over_ranks([sum(gms)], world, dev)
            rec["graph"] = {"us_per_call": g_ms / args.steps * 1e3, "median_us": statistics.median(gms) * 1e3,
                            "value": job_gbs(kvb, world, args.steps, g_ms), "unit": "GB/s"}
            del g
        except Exception as e:  # reported, never fatal
            rec["graph"] = {"error": f"{type(e).__name__}: {e}"[:200]}
        # the same step with the L2 left warm between steps (no flush): whatever share of the
        # step's cache rows fits in the L2 can come from it; compared with the L2's size
        try:
            wev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
            for _ in range(args.warmup):
                step()
            torch.cuda.synchronize(dev)
            for k in range(args.steps):
                step(wev[k])
            torch.cuda.synchronize(dev)
            wms = [e[0].elapsed_time(e[1]) for e in wev]
            (w_ms,) = max_over_ranks([sum(wms)], world, dev)
            l2_bytes = int(torch.cuda.get_device_properties(dev).L2_cache_size)
            rec["warm_l2"] = {"us_per_call": w_ms / args.steps * 1e3, "median_us": statistics.median(wms) * 1e3,
                              "value": job_gbs(kvb, world, args.steps, w_ms), "unit": "GB/s",
                              "kv_bytes_per_call": kvb, "l2_bytes": l2_bytes, "kv_fits_in_l2": kvb <= l2_bytes,
                              "note": "same step, no L2 flush between steps; reported beside the flushed numbers, "
                                      "never as them"}
        except Exception as e:  # reported, never fatal
            rec["warm_l2"] = {"error": f"{type(e).__name__}: {e}"[:200]}

    # end to end through the same public calls with host buffers: pinned inputs copied in,
    # outputs copied out, every step.  The cache itself stays resident (it is the state).
    # The step's host inputs travel in one pinned buffer and one copy (q | block_table |
    # seq_lens, each at a 256-byte boundary), and its results come back in one copy
    # (out | lse): each transfer costs a round trip, whatever its size.
    def _region(nbytes, off):
        return off, off + ((nbytes + 255) // 256) * 256

    q_b, bt_b, sl_b = wl.q.nbytes, wl.block_table.nbytes, wl.seq_lens.nbytes
    q_lo, q_hi = _region(q_b, 0)
    bt_lo, bt_hi = _region(bt_b, q_hi)
    sl_lo, sl_hi = _region(sl_b, bt_hi)
    in_h = torch.zeros(sl_hi, dtype=torch.uint8).pin_memory()
    in_h[q_lo:q_lo + q_b].copy_(torch.from_numpy(wl.q.view(np.uint8).reshape(-1)))
    in_h[bt_lo:bt_lo + bt_b].copy_(torch.from_numpy(wl.block_table.view(np.uint8).reshape(-1)))
    in_h[sl_lo:sl_lo + sl_b].copy_(torch.from_numpy(wl.seq_lens.view(np.uint8).reshape(-1)))
    in_d = torch.empty(sl_hi, dtype=torch.uint8, device=dev)
    q_e = in_d[q_lo:q_lo + q_b].view(torch.bfloat16).view(q.shape)
    bt_e = in_d[bt_lo:bt_lo + bt_b].view(torch.int32).view(bt.shape)
    sl_e = in_d[sl_lo:sl_lo + sl_b].view(torch.int32).view(sl.shape)
    o_b, l_b = out.numel() * 2, lse.numel() * 4
    o_lo, o_hi = _region(o_b, 0)
    l_lo, l_hi = _region(l_b, o_hi)
    res_d = torch.empty(l_hi, dtype=torch.uint8, device=dev)
    out_e = res_d[o_lo:o_lo + o_b].view(torch.bfloat16).view(out.shape)
    lse_e = res_d[l_lo:l_lo + l_b].view(torch.float32).view(lse.shape)
    res_h = torch.empty(l_hi, dtype=torch.uint8).pin_memory()
    e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]

    def e2e_step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        in_d.copy_(in_h, non_blocking=True)
        mla.plan(sl_e, wl.s_q, wl.H, ws, stream=stream)
        mla.decode(q_e, kv, bt_e, sl_e, wl.scale, wl.causal, ws, out_e, lse_e, kv_scale=wl.kv_scale, stream=stream)
        res_h.copy_(res_d, non_blocking=True)
        if ev is not None:
            ev[1].record(stream)

    for _ in range(args.warmup):
        flush_l2(0)
        e2e_step()
    torch.cuda.synchronize(dev)
    for k in range(args.steps):
        flush_l2(k)
        e2e_step(e2e_ev[k])
    torch.cuda.synchronize(dev)
    (e2e_ms,) = max_over_ranks([sum(e[0].elapsed_time(e[1]) for e in e2e_ev)], world, dev)
    rec["e2e"] = {"value": job_gbs(kvb, world, args.steps, e2e_ms), "unit": "GB/s",
                  "h2d_bytes_per_step": int(in_h.numel()), "d2h_bytes_per_step": int(res_h.numel()),
                  "us_per_call": e2e_ms / args.steps * 1e3, "device_step_us": tot_ms / args.steps * 1e3,
                  "note": "q, block_table, seq_lens in (one pinned buffer, one copy) and out, lse back (one copy) "
                          "per step; the paged cache stays resident"}

    def time_op(fn):
        tev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        for _ in range(args.warmup):
            fn()
        for k in range(args.steps):
            flush_l2(k)
            tev[k][0].record(stream)
            fn()
            tev[k][1].record(stream)
        torch.cuda.synchronize(dev)
        return statistics.median(e[0].elapsed_time(e[1]) for e in tev) * 1e3

    if not args.no_side:
        # the write side of the same cache: append the s_q draft rows of each request (rope on
        # the 64-wide key), timed on its own after everything above (it rewrites those rows)
        ckv_new = torch.randn((wl.B, wl.s_q, W.DV), device=dev).to(torch.bfloat16)
        kpe_new = torch.randn((wl.B, wl.s_q, 64), device=dev).to(torch.bfloat16)
        max_pos = int(wl.seq_lens.max()) + 1
        ang = torch.arange(max_pos, device=dev, dtype=torch.float64)[:, None] * \
            (10000.0 ** (-torch.arange(32, device=dev, dtype=torch.float64) / 32.0))[None, :]
        cos_sin = torch.cat([torch.cos(ang), torch.sin(ang)], dim=1).float().contiguous()
        app_us = time_op(lambda: mla.kv_append(ckv_new, kpe_new, cos_sin, kv, bt, sl, kv_scale=wl.kv_scale,
                                               stream=stream))
        elem = 2 if wl.kv_dtype == W.KV_BF16 else 1
        app_bytes = wl.B * wl.s_q * (W.DV * 2 + 64 * 2 + 64 * 4 + W.DQK * elem)
        rec["kv_append"] = {"us_per_call": app_us, "bytes_per_call": app_bytes,
                            "GB/s": app_bytes / (app_us * 1e-6) / 1e9, "rows": wl.B * wl.s_q,
                            "note": "launch-bound at decode sizes; L2 flushed before each call"}
        # the projections on either side of the latent attention, random weights (no model)
        q_nope = torch.randn((wl.B, wl.s_q, wl.H, 128), device=dev).to(torch.bfloat16)
        q_rope = torch.randn((wl.B, wl.s_q, wl.H, 64), device=dev).to(torch.bfloat16)
        w_uk = (torch.randn((wl.H, W.DV, 128), device=dev) / 128 ** 0.5).to(torch.bfloat16)
        w_uv = (torch.randn((wl.H, W.DV, 128), device=dev) / W.DV ** 0.5).to(torch.bfloat16)
        q_abs = torch.empty((wl.B, wl.s_q, wl.H, W.DQK), dtype=torch.bfloat16, device=dev)
        y_proj = torch.empty((wl.B, wl.s_q, wl.H, 128), dtype=torch.bfloat16, device=dev)
        rows = wl.B * wl.s_q * wl.H
        wbytes = wl.H * W.DV * 128 * 2
        ab_us = time_op(lambda: mla.absorb_q(q_nope, q_rope, w_uk, q_abs, stream=stream))
        pj_us = time_op(lambda: mla.project_out(out, w_uv, y_proj, stream=stream))
        ab_bytes = wbytes + rows * (128 + 64 + W.DQK) * 2
        pj_bytes = wbytes + rows * (W.DV + 128) * 2
        proj_flops = 2 * rows * W.DV * 128
        rec["absorb_project"] = {"absorb_q_us": ab_us, "absorb_q_GB/s": ab_bytes / (ab_us * 1e-6) / 1e9,
                                 "project_out_us": pj_us, "project_out_GB/s": pj_bytes / (pj_us * 1e-6) / 1e9,
                                 "flops_each": proj_flops, "absorb_q_tflops": proj_flops / (ab_us * 1e-6) / 1e12,
                                 "project_out_tflops": proj_flops / (pj_us * 1e-6) / 1e12,
                                 "weight_bytes_each": wbytes,
                                 "note": "per-head W_UK / W_UV [H, 512, 128] bf16, L2 flushed before each call"}
    del q, kv, bt, sl, ws, out, lse, in_d, res_d
    torch.cuda.empty_cache()
    return wl, rec


def run_ours(args):
    import torch
    import torch.distributed as dist
    import mla_attention_decode_paged_b200 as mla
    from mla_attention_decode_paged_b200 import build as build_mod

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    build_mod.build(quiet=True)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(256 << 20, dtype=torch.uint8, device=dev).view(torch.int64)

    def flush_l2(k):
        # A 256 MB write (larger than the 126 MB L2), then a 256 MB read of another buffer.
        # The write alone leaves the L2 full of dirty lines, whose write-back would then
        # land inside the next timed kernel (measured: +6 us on agent_spec's scan); the
        # read evicts them here, outside the timed events, and leaves only clean lines.
        flush.fill_(k % 251 + 1)
        flush_rd.sum()

    names = [args.workload] + ([] if args.only else [n for n in W.WORKLOAD_ORDER if n != args.workload])
    recs = {}
    head_wl = None
    for n in names:
        wl, rec = measure_workload(n, args, dev, stream, flush_l2, world, headline=(n == args.workload))
        recs[n] = rec
        if n == args.workload:
            head_wl = wl
    head = recs[args.workload]

    def time_op(fn):
        tev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        for _ in range(args.warmup):
            fn()
        for k in range(args.steps):
            flush_l2(k)
            tev[k][0].record(stream)
            fn()
            tev[k][1].record(stream)
        torch.cuda.synchronize(dev)
        return statistics.median(e[0].elapsed_time(e[1]) for e in tev) * 1e3

    prefill_line = None
    if not args.no_side:
        try:
            prefill_line = prefill_measure(args, dev, stream, flush_l2, time_op)
        except (RuntimeError, mla.MlaError) as e:  # reported in the line; the decode numbers stand
            prefill_line = {"error": str(e)}

    wl = head_wl
    line = {"metric": METRIC, "value": head["value"], "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": head["us_per_call"] * 1e-3, "us_per_call": head["us_per_call"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if wl.kv_dtype == W.KV_BF16 else "e4m3->bf16",
            "data": "synthetic (seeded N(0,1) q/KV; no dataset)",
            "config": {"workload": head["workload"], "global_batch": wl.B * world, "seq_len": int(wl.seq_lens.max()),
                       "parallelism": f"replicas x{world} (no collective)",
                       "l2": "flushed between steps outside the timed events: a 256 MB write, then a 256 MB read that evicts its dirty lines"},
            "breakdown_us": head["breakdown_us"], "tflops": head["tflops"],
            "roofline_us": head["roofline_us"], "frac_of_roofline_step": head["frac_of_roofline_step"],
            "roofline": head["roofline"], "roofline_nominal": head["roofline_nominal"],
            "step_us_p10_p50_p90": head["step_us_p10_p50_p90"],
            "graph": head.get("graph"), "warm_l2": head.get("warm_l2"), "e2e": head["e2e"],
            "kv_append": head.get("kv_append"), "absorb_project": head.get("absorb_project"),
            "prefill": prefill_line,
            "workloads": {n: {k: v for k, v in r.items() if k not in ("graph", "warm_l2")} for n, r in recs.items()},
            "gpu_launches": 3 * args.steps,
            "gpu_launches_note": "plan + split scan + combine per timed step of the headline workload",
            "clocks": head["clocks"]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        full_s, cores, desc = oracle_baseline(wl)
        line["cpu_baseline"] = {"value": wl.kv_bytes() / full_s / 1e9, "unit": "GB/s", "cores": cores,
                                "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(W.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--soak-s", type=float, default=1.0, help="untimed identical steps around the timed ones")
    ap.add_argument("--only", action="store_true", help="measure the headline workload alone")
    ap.add_argument("--no-side", action="store_true", help="skip the KV append, projection and prefill timings")
    ap.add_argument("--tokens", type=int, default=None,
                    help="every request this many tokens (a reduced case for profiler captures; the line's "
                         "config says so)")
    args = ap.parse_args()
    if args.warmup < 3:
        log("warmup raised to 3 (minimum)")
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
