#!/usr/bin/env python
"""Valid-token attention TFLOP/s of sigmoid attention over a padded variable-length batch.

One step = the whole hot path on one batch: forward (sigattn_fwd) and backward
(sigattn_bwd: the dK/dV kernel, then the dQ kernel; plus the D preprocess in the softmax
modes), with the tile plan built once per batch beforehand (it is shared by every head and
layer; its build time is reported separately as plan_ms).  FLOPs counted on valid
(query, key) pairs P only: forward 4 d H P, backward 2.5x forward.

Default workload: the single-cell batch (B=32, lengths log-uniform in [200, 2048] padded
to the batch max, H=8, d=64, sigmoid with b = -log n).

    python bench.py [--gpus N --steps K --warmup W --config {1..5} --epilogue E]
    python bench.py --impl reference ...   # the float64 CPU oracle on the host cores

Prints one JSON line (rank 0).  Multi-GPU (torchrun): independent replicas, one batch per
rank, no collective on the data path; the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from padded_variable_length_b200 import workloads as W  # noqa: E402
from padded_variable_length_b200.replicas import (  # noqa: E402
    job_throughput, max_over_ranks, replica_seed)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
EPI_BY_NAME = {"sigmoid": W.SIGMOID, "softmax": W.SOFTMAX, "softmax1": W.SOFTMAX1}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_name(w: W.Workload, epi: int) -> str:
    if w.lengths is not None:
        desc = (f"{w.name}: B={w.B} padded to {w.Nq}, lengths {int(w.lengths.min())}..{int(w.lengths.max())}"
                f" (sum n^2 = {w.pairs()}), H={w.H}, d={w.d}")
    else:
        desc = f"{w.name}: B={w.B}, N={w.Nq}, element mask with {w.pairs()} pairs, H={w.H}, d={w.d}"
    return f"{desc}, {W.EPILOGUE_NAMES[epi]}, seed {w.seed}"


def bench_workload(args, epi: int) -> W.Workload:
    """The workload of --config, or of --mask (the other block-mask families); --batch keeps
    only its first batch entries (a smaller case of the same shapes, for profiler captures)."""
    w = W.mask_family(args.mask, epilogue=epi) if args.mask else W.config(args.config, epilogue=epi)
    if args.batch and args.batch < w.B:
        nb = args.batch
        if w.lengths is not None:
            w = W.padded_workload(w.name, w.lengths[:nb], H=w.H, d=w.d, epilogue=epi, backward=True,
                                  seed=w.seed, npad=w.Nq)
        else:
            w = W.masked_workload(w.name, w.mask[:nb], w.counts[:nb], H=w.H, d=w.d, epilogue=epi,
                                  backward=True, seed=w.seed,
                                  doc_lengths=w.doc_lengths[:nb] if w.doc_lengths else None)
    return w


def fwd_flops(w: W.Workload) -> float:
    return 4.0 * w.d * w.H * w.pairs()


# ------------------------------------------------------------------------------------------
# clocks
# ------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------------------------------------
# the oracle on the host cores (CPU baseline and the reference arm)
# ------------------------------------------------------------------------------------------
def oracle_sample(w: W.Workload, epi: int, t: dict, pairs_bh, budget_s: float):
    """Runs the float64 oracle forward + backward on (b, h) pairs in order until the time
    budget is spent; returns (flops done, seconds, pairs done)."""
    from oracle import attention as A
    bias = A.bias_from_counts(w.counts) if epi == W.SIGMOID else np.zeros((w.B, w.Nq))
    mp = A.mask_provider(w.lengths, w.mask, w.Nq, w.Nk)
    scale = 1.0 / math.sqrt(w.d)
    done, flops = 0, 0.0
    t0 = time.perf_counter()
    for (b, h) in pairs_bh:
        q = t["q"][b, :, h].double().numpy()
        k = t["k"][b, :, h].double().numpy()
        v = t["v"][b, :, h].double().numpy()
        do = t["do"][b, :, h].double().numpy()
        mr = mp(b)
        o, _ = A.head_forward(q, k, v, mr, bias[b], scale, epi)
        A.head_backward(q, k, v, do, mr, bias[b], scale, epi, o=o)
        pairs = int(w.lengths[b]) ** 2 if w.lengths is not None else int(w.mask[b].astype(np.int64).sum())
        flops += 3.5 * 4.0 * w.d * pairs
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    return flops, time.perf_counter() - t0, done


def cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return None
    epi = EPI_BY_NAME[args.epilogue]
    w = bench_workload(args, epi)
    w.backward = True
    t = W.tensors(w, with_grad=True)
    order = [(b, h) for h in range(w.H) for b in range(w.B)]
    for i in range(args.warmup):
        oracle_sample(w, epi, t, [order[i % len(order)]], 1e9)
    flops, secs = 0.0, 0.0
    for i in range(args.steps):
        f, s, _ = oracle_sample(w, epi, t, [order[(args.warmup + i) % len(order)]], 1e9)
        flops += f
        secs += s
    value = flops / secs / 1e12
    sample = f"one (batch entry, head) pair of the workload per step, forward + backward in float64"
    return {
        "metric": "valid-token attention TFLOP/s (fwd+bwd)", "value": value, "unit": "TFLOP/s",
        "impl": "reference", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(w, epi)},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------------------------------
# the CUDA path
# ------------------------------------------------------------------------------------------
def run_ours(args, rank: int, world: int, local_rank: int):
    from padded_variable_length_b200 import binding as Bd
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    epi = EPI_BY_NAME[args.epilogue]
    w = bench_workload(args, epi)
    w.backward = True
    w.seed = replica_seed(w.seed, rank)
    t = W.tensors(w, with_grad=True)
    stream = torch.cuda.current_stream()
    d = {k: v.to(dev) for k, v in t.items()}
    counts = torch.from_numpy(np.ascontiguousarray(w.counts, dtype=np.int32)).to(dev)

    # the planner's input, resident on the device before its timing starts
    plan_in = (torch.from_numpy(w.lengths.astype(np.int32)).to(dev) if w.lengths is not None
               else torch.from_numpy(w.mask).to(dev))

    def build_plan():
        if w.lengths is not None:
            return Bd.Plan.from_lengths(plan_in, w.Nq)
        return Bd.Plan.from_mask(plan_in)

    # plan build time (reported, not part of the step): median of 15 builds, each bracketed
    # by events on the stream (a lengths or mask build returns without waiting for the
    # device, so the events span its kernels and the host time before the first of them)
    for _ in range(3):
        build_plan().close()
    torch.cuda.synchronize()
    plan_times = []
    for _ in range(15):
        pe0, pe1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        pe0.record(stream)
        p_ = build_plan()
        pe1.record(stream)
        torch.cuda.synchronize()
        plan_times.append(pe0.elapsed_time(pe1))
        p_.close()
    plan_ms = statistics.median(plan_times)
    plan = build_plan()
    sizes = plan.sizes()

    bias = Bd.bias_from_counts(counts) if epi == W.SIGMOID else None
    o = torch.empty_like(d["q"])
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev) if epi != W.SIGMOID else None
    ws = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev) if epi != W.SIGMOID else None
    dq, dk, dv = torch.empty_like(d["q"]), torch.empty_like(d["k"]), torch.empty_like(d["v"])
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)  # 256 MB > L2

    fused = args.bwd == "fused" or (args.bwd == "auto" and w.d == 64)
    fwd_part = lambda: Bd.fwd(plan, d["q"], d["k"], d["v"], bias, epi, out=o, lse=lse)
    if fused:
        fws = torch.empty((Bd.bwd_fused_workspace_bytes(plan, w.H, w.d, epi) + 3) // 4,
                          dtype=torch.float32, device=dev)
        parts = [fwd_part,
                 lambda: Bd.bwd_fused(plan, d["q"], d["k"], d["v"], o, d["do"], bias, epi, lse=lse,
                                      workspace=fws, dq=dq, dk=dk, dv=dv)]
        part_names = ["fwd", "bwd_fused"]
        # forward; [D preprocess,] accumulator zeroing, fused kernel, dQ conversion
        launches_per_step = 1 + 3 + (1 if epi != W.SIGMOID else 0)
    else:
        parts = [fwd_part,
                 lambda: Bd.bwd(plan, d["q"], d["k"], d["v"], o, d["do"], bias, epi, lse=lse,
                                workspace=ws, dq=dq, dk=dk, dv=dv, parts=Bd.BWD_PREP | Bd.BWD_DKDV),
                 lambda: Bd.bwd(plan, d["q"], d["k"], d["v"], o, d["do"], bias, epi, lse=lse,
                                workspace=ws, dq=dq, dk=dk, dv=dv, parts=Bd.BWD_DQ)]
        part_names = ["fwd", "bwd_dkdv", "bwd_dq"]
        launches_per_step = 3 + (1 if epi != W.SIGMOID else 0)
    if not args.no_graph:
        # One CUDA graph per part: the host only replays, so no launch preparation (tensor
        # maps, argument checks, Python) sits between the device events.
        for fn in parts:
            fn()
        torch.cuda.synchronize()
        graphs = []
        for fn in parts:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            graphs.append(g)
        torch.cuda.synchronize()
        parts = [g.replay for g in graphs]

    L_ = args.layers  # layers per step, all on the one plan (built once per batch)

    def step(ev=None):
        for layer in range(L_):
            for k_, fn in enumerate(parts):
                if ev:
                    ev[layer * len(parts) + k_].record(stream)
                fn()
        if ev:
            ev[L_ * len(parts)].record(stream)

    sampler = ClockSampler(local_rank if os.environ.get("CUDA_VISIBLE_DEVICES") is None else 0)
    sampler.start()
    t_warm = time.perf_counter()
    while True:  # warm-up: at least W steps and ~0.5 s so the clock sampler sees load
        for _ in range(max(1, args.warmup)):
            step()
            flush.zero_()
        torch.cuda.synchronize()
        if time.perf_counter() - t_warm > 0.5:
            break
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(L_ * len(parts) + 1)]
           for _ in range(args.steps)]
    for i in range(args.steps):
        step(evs[i])
        flush.zero_()  # L2 flush between timed steps (outside the events)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    assert Bd.get_status() == 0, "device status reports a timed-out wait"
    # per part, summed over steps and layers; the per-launch figures below divide by both
    part_ms = [sum(e[layer * len(parts) + k_].elapsed_time(e[layer * len(parts) + k_ + 1])
                   for e in evs for layer in range(L_)) / L_ for k_ in range(len(parts))]
    total_ms = max_over_ranks(sum(e[0].elapsed_time(e[-1]) for e in evs), dev)

    ff = fwd_flops(w)
    step_flops = 3.5 * ff * L_
    value = job_throughput(world, step_flops, args.steps, total_ms)
    peaks, peak_src = load_peaks()
    peak_tf = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    K = args.steps
    # algorithmic FLOPs of each part: forward 4 d per pair; backward 10 d per pair, of
    # which dK / dV 8 d and dQ 2 d in the split form
    part_flops = {"fwd": ff, "bwd_fused": 2.5 * ff, "bwd_dkdv": 2.0 * ff, "bwd_dq": 0.5 * ff}
    kernels = {}
    for name, ms in zip(part_names, part_ms):
        kernels[name] = {"ms": ms / K, "flops": part_flops[name],
                         "tflops": part_flops[name] / (ms / K / 1e3) / 1e12}
    bwd_ms = sum(part_ms[1:])
    dom = max(kernels, key=lambda k: kernels[k]["ms"])
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath):
        with open(tpath) as f:
            tr = json.load(f)
        # the mask families and the reduced (--batch) captures have no entry of their own
        key = f"{dom}|{args.mask or args.config}|{args.epilogue}"
        traffic = None if args.batch else tr.get(key)
    roofline = {"bound": "tensor", "kernel": dom, "achieved": kernels[dom]["tflops"],
                "peak": peak_tf, "unit": "TFLOP/s", "frac": kernels[dom]["tflops"] / peak_tf,
                "peak_source": f"{peak_src} burst bf16 (cuBLAS)", "traffic": traffic}
    # the forward's rate against HBM: algorithmic bytes = read Q, K, V and write O once over
    # the valid tokens (8 bytes per token, head and channel)
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    fwd_bytes = 8.0 * w.valid_tokens() * w.H * w.d
    kernels["fwd"]["bytes"] = fwd_bytes
    kernels["fwd"]["gb_per_s"] = fwd_bytes / (kernels["fwd"]["ms"] * 1e-3) / 1e9
    if args.config == 1 and not args.mask:
        # a handful of tiles: no contraction to speak of, the bound is memory and latency
        roofline = {"bound": "hbm", "kernel": "fwd", "achieved": kernels["fwd"]["gb_per_s"],
                    "peak": hbm, "unit": "GB/s", "frac": kernels["fwd"]["gb_per_s"] / hbm,
                    "peak_source": f"{peak_src} copy", "traffic": traffic}

    out = {
        "metric": "valid-token attention TFLOP/s (fwd+bwd)", "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": total_ms / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": workload_name(w, epi), "l2": "flushed (256 MB write) between steps",
                   "plan": "built once per batch, outside the step",
                   "layers_per_step": L_,
                   "launch": "API calls each step" if args.no_graph else "CUDA graph replay per part",
                   "parallelism": f"{world} independent replicas" if world > 1 else "1 GPU"},
        "fwd_tflops": kernels["fwd"]["tflops"], "fwd_frac": kernels["fwd"]["tflops"] / peak_tf,
        "bwd_tflops": 2.5 * ff / (bwd_ms / K / 1e3) / 1e12,
        "bwd_frac": 2.5 * ff / (bwd_ms / K / 1e3) / 1e12 / peak_tf,
        "bwd_algo": "fused (one kernel, dQ by TMA reduce-add)" if fused else "split (dK/dV + dQ)",
        "kernels": kernels, "plan_ms": plan_ms, "layers": L_,
        "plan_share": plan_ms / (plan_ms + total_ms / K),
        "plan": plan_report(w, plan_ms, peaks, peak_src),
        "tiles": {"nonempty": sizes["nonempty"], "full": sizes["full"], "partial": sizes["partial"],
                  "grid_total": sizes["grid_total"],
                  "skipped_frac": 1.0 - sizes["nonempty"] / max(1, sizes["grid_total"])},
        "roofline": roofline,
        "gpu_launches": launches_per_step * K,
        "clocks": clocks,
    }

    # ---- end to end through the C ABI with host buffers (pinned), copies inside the timing
    out["e2e"] = run_e2e(Bd, w, t, epi, dev, stream, args, world, fused)
    packed = run_e2e_packed(Bd, w, t, epi, dev, stream, args, world, fused)
    if packed is not None:
        out["e2e_packed"] = packed
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        order = [(b, h) for h in range(w.H) for b in range(w.B)]
        f, s, n = oracle_sample(w, epi, t, order, args.cpu_seconds)
        out["cpu_baseline"] = {
            "value": f / s / 1e12, "unit": "TFLOP/s", "cores": cores(), "kind": "oracle",
            "sample": f"{n} of {len(order)} (batch entry, head) pairs of this workload, float64 "
                      f"forward + backward, {s:.1f} s on the host"}
    plan.close()
    return out


def plan_report(w, plan_ms, peaks, peak_src):
    """The planner's rate: an element mask is read once (1 byte per element; the PARTIAL
    blocks' bytes a second time for their bitmasks), a lengths plan reads B ints."""
    if w.mask is not None:
        nbytes = int(w.mask.size)
        gbs = nbytes / (plan_ms * 1e-3) / 1e9
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        return {"input": "element mask", "bytes": nbytes, "ms": plan_ms, "gb_per_s": gbs,
                "hbm_frac": gbs / hbm, "hbm_peak_gbs": hbm, "peak_source": f"{peak_src} copy"}
    return {"input": "lengths", "bytes": int(w.lengths.size * 4), "ms": plan_ms}


def timed_two_streams(step, steps, stream, dev, warm=4):
    """Runs `steps` calls of step() alternately on two streams (so that one step's
    device-to-host copies overlap the next step's host-to-device copies on the full-duplex
    link) and returns the device time from before the first to after the last, in ms.
    `warm` untimed calls on the same two streams come first (the caching allocator keeps
    device memory per stream)."""
    pair = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
    for i in range(warm):
        with torch.cuda.stream(pair[i % 2]):
            step(i % 2).close()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s_ in pair:
        s_.wait_event(e0)
    plans = []
    for i in range(steps):
        with torch.cuda.stream(pair[i % 2]):
            plans.append(step(i % 2))
    for s_ in pair:
        done = torch.cuda.Event()
        done.record(s_)
        stream.wait_event(done)
    e1.record(stream)
    torch.cuda.synchronize()
    for p in plans:
        p.close()
    return e0.elapsed_time(e1)


def run_e2e(Bd, w, t, epi, dev, stream, args, world, fused):
    """Same metric through the user's call with HOST buffers: every step copies Q, K, V, dO,
    the lengths (or mask) and the bias counts in from pinned memory, builds the plan, runs
    forward + backward, and copies O, dQ, dK, dV back out."""
    pin = {k: v.pin_memory() for k, v in t.items()}
    host_lengths = (torch.from_numpy(w.lengths.astype(np.int32)).pin_memory()
                    if w.lengths is not None else None)
    host_mask = torch.from_numpy(w.mask).pin_memory() if w.mask is not None else None
    host_counts = torch.from_numpy(np.ascontiguousarray(w.counts, dtype=np.int32)).pin_memory()
    # one set of host result buffers per stream (two steps are in flight at once)
    outs2 = []
    for _ in range(2):
        outs = {k: torch.empty_like(pin["q"]).pin_memory() for k in ("o", "dq")}
        outs.update({k: torch.empty_like(pin["k"]).pin_memory() for k in ("dk", "dv")})
        outs2.append(outs)
    h2d = sum(x.numel() * x.element_size() for x in pin.values()) + host_counts.numel() * 4
    h2d += host_lengths.numel() * 4 if host_lengths is not None else host_mask.numel()
    d2h = sum(x.numel() * x.element_size() for x in outs2[0].values())

    def e2e_step(par=0):
        outs = outs2[par]
        d = {k: v.to(dev, non_blocking=True) for k, v in pin.items()}
        counts = host_counts.to(dev, non_blocking=True)
        if host_lengths is not None:
            plan = Bd.Plan.from_lengths(host_lengths.to(dev, non_blocking=True), w.Nq)
        else:
            plan = Bd.Plan.from_mask(host_mask.to(dev, non_blocking=True))
        bias = Bd.bias_from_counts(counts) if epi == W.SIGMOID else None
        o, lse = Bd.fwd(plan, d["q"], d["k"], d["v"], bias, epi)
        bwd = Bd.bwd_fused if fused else Bd.bwd
        dq, dk, dv = bwd(plan, d["q"], d["k"], d["v"], o, d["do"], bias, epi, lse=lse)
        for name, x in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv)):
            outs[name].copy_(x, non_blocking=True)
        return plan

    steps = max(3, min(args.steps, 10))
    ms = max_over_ranks(timed_two_streams(e2e_step, steps, stream, dev), dev)
    value = job_throughput(world, 3.5 * fwd_flops(w), steps, ms)
    return {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": steps, "ms_per_step": ms / steps,
            "streams": "two, alternating steps (copies of consecutive steps overlap)"}


def run_e2e_packed(Bd, w, t, epi, dev, stream, args, world, fused):
    """The e2e leg with PACKED host buffers (valid tokens only, sequence b at rows cu[b]..):
    every step copies the packed Q, K, V, dO, the cumulative offsets and the per-row counts
    in, builds the plan from the offsets, runs forward + backward on the packed layout, and
    copies the packed O, dQ, dK, dV out.  Same valid-token FLOPs as the padded leg."""
    if w.lengths is None:
        return None
    lengths = w.lengths.astype(np.int64)
    pk = {k: torch.cat([v[b, :int(n)] for b, n in enumerate(lengths)], 0).contiguous().pin_memory()
          for k, v in t.items()}
    cu = torch.from_numpy(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)).pin_memory()
    counts = torch.from_numpy(np.repeat(lengths, lengths).astype(np.int32)).pin_memory()
    outs2 = [{k: torch.empty_like(pk["q"]).pin_memory() for k in ("o", "dq", "dk", "dv")}
             for _ in range(2)]  # one set per stream
    h2d = sum(x.numel() * x.element_size() for x in pk.values()) + cu.numel() * 4 + counts.numel() * 4
    d2h = sum(x.numel() * x.element_size() for x in outs2[0].values())
    maxlen = int(lengths.max())

    def step(par=0):
        outs = outs2[par]
        d = {k: v.to(dev, non_blocking=True) for k, v in pk.items()}
        plan = Bd.Plan.from_cu_seqlens(cu.to(dev, non_blocking=True), maxlen)
        bias = Bd.bias_from_counts(counts.to(dev, non_blocking=True)) if epi == W.SIGMOID else None
        o, lse = Bd.fwd(plan, d["q"], d["k"], d["v"], bias, epi)
        bwd = Bd.bwd_fused if fused else Bd.bwd
        dq, dk, dv = bwd(plan, d["q"], d["k"], d["v"], o, d["do"], bias, epi, lse=lse)
        for name, x in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv)):
            outs[name].copy_(x, non_blocking=True)
        return plan

    steps = max(3, min(args.steps, 10))
    ms = max_over_ranks(timed_two_streams(step, steps, stream, dev), dev)
    value = job_throughput(world, 3.5 * fwd_flops(w), steps, ms)
    return {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": steps, "ms_per_step": ms / steps,
            "layout": "packed host buffers (valid tokens only), plan from cumulative offsets",
            "streams": "two, alternating steps (copies of consecutive steps overlap)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=2, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--epilogue", default="sigmoid", choices=list(EPI_BY_NAME))
    ap.add_argument("--mask", default=None, choices=["longformer", "tree", "packed"],
                    help="run a block-mask family (B=4, H=16, d=128) instead of --config")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--bwd", default="auto", choices=["auto", "fused", "split"],
                    help="backward form: fused (d = 64 only) or the two-kernel split; auto = "
                         "fused where supported")
    ap.add_argument("--batch", type=int, default=0,
                    help="keep only the first B batch entries of the workload (profiling)")
    ap.add_argument("--layers", type=int, default=1,
                    help="attention layers per step, all reusing the one plan of the batch")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every part through the API each step instead of replaying CUDA graphs")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    if args.impl == "reference":
        out = run_reference(args, rank, world)
    else:
        out = run_ours(args, rank, world, local_rank)
    if world > 1 and args.impl == "ours":
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0 and out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
