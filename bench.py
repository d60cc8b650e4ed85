#!/usr/bin/env python
"""Benchmark of the bf16 (shifted-)window attention layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl vswin|reference]

A step is one pass of the whole layer path over one batch: for the headline
workload (Swin-T stage 1, 32x224^2 clips, batch 8) the W-MSA layer and the
SW-MSA layer of a block pair, each on the (8, 16, 56, 56, 96) token tensor.
Inputs are synthetic and seeded, resident in HBM before timing; L2 is flushed
by a 512 MB write before every timed step (outside the step's events).

One JSON line is printed by rank 0. ``value`` is layer-tokens per second for
the whole job (every token passes through both layers of the pair), timed with
CUDA events, the slowest rank's time over the sum of all ranks' tokens. With
``--impl reference`` the double-precision CPU oracle is timed instead, on a
bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from shifted_window_attention_sw_b200 import replicas  # noqa: E402
from shifted_window_attention_sw_b200.accounting import layer_work  # noqa: E402
from shifted_window_attention_sw_b200.inputs import workload_layer_inputs  # noqa: E402
from shifted_window_attention_sw_b200.workloads import HEADLINE, WORKLOADS  # noqa: E402

METRIC = "SW-MSA layer tokens/s and TFLOP/s (frac of bf16 peak), Swin-T stage1 32×224² b8"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLUSH_BYTES = 512 << 20


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"


def cpu_model():
    """The host CPU's model name (first processor in /proc/cpuinfo), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


# The MUFU (special-function unit) rate of sm_100: 16 ex2 results per clock per SM.
MUFU_EX2_PER_CLK_SM = 16
SMS = 148


def exp_bound_us(exps, sm_mhz):
    """Time the exponentials alone need on the MUFU at the given SM clock."""
    return exps / (SMS * MUFU_EX2_PER_CLK_SM * sm_mhz * 1e6) * 1e6


def workload_config(wl):
    layers = []
    for ly in wl.layers:
        layers.append({"B": ly.B, "T": ly.T, "H": ly.H, "W": ly.W, "C": ly.C, "heads": ly.heads,
                       "window": list(ly.window), "shift": list(ly.shift)})
    return {"workload": wl.name, "description": wl.description, "layers": layers,
            "tokens_per_layer": wl.layers[0].B * wl.layers[0].T * wl.layers[0].H * wl.layers[0].W,
            "l2": "flushed by a 512 MB write before every timed step", "parallelism": "replicas"}


def step_work(wl):
    tot = {"tokens": 0, "flops": 0, "attn_flops": 0, "gemm_flops": 0, "bytes": 0, "exps": 0,
           "unmasked_pairs": 0, "pairs": 0}
    for ly in wl.layers:
        w = layer_work(ly.B, ly.T, ly.H, ly.W, ly.C, ly.heads, ly.window, ly.shift, 2)
        for k in tot:
            tot[k] += w[k]
    return tot


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and throttle reasons DURING the timed region with nvidia-smi in a
    separate process (-lms period), so nothing runs inside the benchmark process."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device, period_ms=50):
        self.proc = None
        self.period_ms = period_ms
        props = torch.cuda.get_device_properties(device)
        self.bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"

    def start(self):
        import subprocess

        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.bus}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 f"-lms={self.period_ms}"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)  # let the first sample land before the timed region starts
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, reasons = [], None, set()
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 6:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            for name, v in zip(self.NAMES, f[2:6]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": float(statistics.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle sample
def oracle_sample(wl, target_s, nthreads=0, layers=None):
    """Time the CPU oracle on a bounded sample of the workload: whole windows of each
    layer (forward_windows), as many as fit in about target_s seconds."""
    import oracle

    oracle.build()
    cores = oracle.max_threads(nthreads)
    layers = layers if layers is not None else wl.layers
    inputs = [workload_layer_inputs(wl, ly, scale="baseline").as_f64() for ly in layers]
    # window maps (to count real tokens) are computed once, outside the timed region
    geoms = [oracle.geometry(ly.T, ly.H, ly.W, ly.window, ly.shift) for ly in layers]
    srcs = [oracle.index_maps(ly.B, ly.T, ly.H, ly.W, ly.window, ly.shift)[0] for ly in layers]

    def run(nwin_per_layer):
        tokens, dt = 0, 0.0
        for ly, a, g, src in zip(layers, inputs, geoms, srcs):
            total = ly.B * g["nW"]
            wins = np.linspace(0, total - 1, num=min(nwin_per_layer, total)).astype(np.int64)
            t0 = time.perf_counter()
            oracle.forward_windows(a["x"], ly.window, ly.shift, a["Wqkv"], a["bqkv"], a["Wproj"], a["bproj"],
                                   a["table"], ly.heads, wins, nthreads=nthreads)
            dt += time.perf_counter() - t0
            N = g["N"]
            tokens += int(sum((src[w * N:(w + 1) * N] >= 0).sum() for w in wins))
        return tokens, dt

    # calibration: start with one window per thread and layer, then scale the
    # sample until the timed oracle work is at least half the target
    n = cores
    tok, dt = run(n)
    total = max(ly.B * g["nW"] for ly, g in zip(layers, geoms))
    for _ in range(4):
        if dt >= 0.5 * target_s or n >= total:
            break
        n = min(total, max(n + 1, int(n * min(8.0, target_s / max(dt, 1e-6)))))
        tok, dt = run(n)
    return {"tokens": tok, "seconds": dt, "cores": cores, "windows_per_layer": n}


def run_reference(args):
    rank, world, _ = replicas.env_rank()
    if rank != 0:
        return 0
    wl = WORKLOADS[args.workload]
    import oracle

    oracle.build()
    cores = oracle.max_threads(0)
    budget = max(2.0, 150.0 / max(1, args.steps + args.warmup))
    # calibrate the per-step sample so the whole run stays within a few minutes
    cal = oracle_sample(wl, budget)
    nwin = cal["windows_per_layer"]
    _oracle_prep(wl, nwin)  # inputs and window maps, outside the timed steps
    times, toks = [], 0
    for k in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        s = _oracle_fixed(wl, nwin)
        dt = time.perf_counter() - t0
        if k >= args.warmup:
            times.append(dt)
            toks += s
    total = sum(times)
    value = toks / total
    work = step_work(wl)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": 0,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl),
        "tflops": value * work["flops"] / work["tokens"] / 1e12,
        "cpu_baseline": {"kind": "oracle", "value": value, "unit": "tokens/s", "cores": cores,
                         "cpu_model": cpu_model(),
                         "sample": f"{nwin} whole windows of each layer per step (evenly spaced), "
                                   f"double precision, OpenMP over windows"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


_ORACLE_CACHE = {}


def _oracle_fixed(wl, nwin):
    """One reference-arm step: the oracle on `nwin` evenly spaced whole windows of each
    layer; returns the real (non-padding) tokens of those windows. Inputs, window maps
    and token counts are prepared once per workload and sample size, outside the
    timed call."""
    import oracle

    tokens = 0
    for ly, a, wins, tok in _oracle_prep(wl, nwin):
        oracle.forward_windows(a["x"], ly.window, ly.shift, a["Wqkv"], a["bqkv"], a["Wproj"], a["bproj"],
                               a["table"], ly.heads, wins)
        tokens += tok
    return tokens


def _oracle_prep(wl, nwin):
    import oracle

    key = (wl.name, nwin)
    if key not in _ORACLE_CACHE:
        prep = []
        for ly in wl.layers:
            a = workload_layer_inputs(wl, ly, scale="baseline").as_f64()
            g = oracle.geometry(ly.T, ly.H, ly.W, ly.window, ly.shift)
            total = ly.B * g["nW"]
            wins = np.linspace(0, total - 1, num=min(nwin, total)).astype(np.int64)
            src, _, _ = oracle.index_maps(ly.B, ly.T, ly.H, ly.W, ly.window, ly.shift)
            N = g["N"]
            tok = int(sum((src[w * N:(w + 1) * N] >= 0).sum() for w in wins))
            prep.append((ly, a, wins, tok))
        _ORACLE_CACHE[key] = prep
    return _ORACLE_CACHE[key]


# ------------------------------------------------------------------ GPU arm
def traffic_record(kernel, workload):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if the counters
    were taken on `workload` and the kernel source has not changed since (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    entry = rec.get(kernel)
    if not entry or entry.get("workload") != workload:
        return None
    src = os.path.join(ROOT, "shifted_window_attention_sw_b200", "csrc", entry.get("source", ""))
    try:
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
    except OSError:
        return None
    if digest != entry.get("sha256"):
        return None
    return entry


def run_gpu(args):
    from shifted_window_attention_sw_b200 import build as build_mod
    from shifted_window_attention_sw_b200 import vswin

    rank, world = replicas.init("nccl")
    _, _, local = replicas.env_rank()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if rank == 0:
        build_mod.build()
    replicas.barrier(device)
    vswin.lib()
    wl = WORKLOADS[args.workload]
    layers = wl.layers
    ins = [workload_layer_inputs(wl, ly, scale="baseline").to(device) for ly in layers]
    outs = [torch.empty_like(i.x) for i in ins]
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        for ly, i, o in zip(layers, ins, outs):
            vswin.wmsa_forward(i.x, ly.window, ly.shift, i.Wqkv, i.bqkv, i.Wproj, i.bproj, i.table, ly.heads,
                               out=o, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(device)
    if vswin.poll_error(stream) != vswin.OK:
        raise RuntimeError("kernel error during warm-up: " + vswin.last_error())

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(device)
    replicas.barrier(device)
    torch.cuda.synchronize(device)
    launches0 = vswin.launch_count()
    vswin.profile_enable(True)
    sampler.start()
    for k in range(args.steps):
        flush.zero_()
        evs[k][0].record(stream)
        step()
        evs[k][1].record(stream)
    torch.cuda.synchronize(device)
    clocks = sampler.stop()
    replicas.barrier(device)
    vswin.profile_enable(False)
    prof = vswin.profile_collect()
    launches = vswin.launch_count() - launches0
    status = vswin.poll_error(stream)
    if status != vswin.OK:
        raise RuntimeError("kernel error in the timed region: " + vswin.last_error())
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_s = sum(step_ms) / 1e3
    # the same steps with L2 left warm (no flush between steps): the inputs of one layer
    # (77 MB) fit in the 126 MB L2, so this is the best case the cold number is bounded by
    n_warm = max(1, min(args.steps, 20))
    w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    step()
    w0.record(stream)
    for _ in range(n_warm):
        step()
    w1.record(stream)
    torch.cuda.synchronize(device)
    warm_s = w0.elapsed_time(w1) / 1e3
    step_stats = {"min": min(step_ms), "median": statistics.median(step_ms), "max": max(step_ms)}
    work = step_work(wl)
    max_s, tokens, nranks = replicas.combine(total_s, work["tokens"] * args.steps, device)
    value = tokens / max_s
    warm_max_s, warm_tokens, _ = replicas.combine(warm_s, work["tokens"] * n_warm, device)
    tflops = nranks * work["flops"] * args.steps / max_s / 1e12

    # end to end through the host-buffer entry point: H2D of x and D2H of out inside the timing
    e2e = None
    if not args.no_e2e:
        xh = [i.x.cpu().pin_memory() for i in ins]
        oh = [torch.empty_like(x).pin_memory() for x in xh]
        n_e2e = max(1, min(args.steps, 10))

        def e2e_step():
            for ly, i, x, o in zip(layers, ins, xh, oh):
                vswin.wmsa_forward_host(x, ly.window, ly.shift, i.Wqkv, i.bqkv, i.Wproj, i.bproj, i.table,
                                        ly.heads, o, stream=stream)

        e2e_step()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        replicas.barrier(device)
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(device)
        e_s = e0.elapsed_time(e1) / 1e3
        e_max, e_tok, _ = replicas.combine(e_s, work["tokens"] * n_e2e, device)
        e2e = {"value": e_tok / e_max, "unit": "tokens/s",
               "h2d_bytes_per_step": int(sum(x.numel() * x.element_size() for x in xh)),
               "d2h_bytes_per_step": int(sum(o.numel() * o.element_size() for o in oh)),
               "steps": n_e2e, "api": "vswin_wmsa_forward_host (pinned host buffers)"}

    if rank != 0:
        replicas.shutdown()
        return 0

    peaks, peak_src = load_peaks()
    # dominant kernel by device time
    dom = max(("qkv_gemm", "attention", "proj_gemm"), key=lambda k: prof[k][0])
    dom_ms, dom_launches = prof[dom]
    if dom == "attention":
        dom_work, unit, bound = work["attn_flops"] * args.steps, "TFLOP/s", "tensor"
        achieved = dom_work / dom_launches / (dom_ms / dom_launches / 1e3) / 1e12
        peak = float(peaks["bf16_tflops"])
        traffic_kernel = "attention_kernel"
    else:
        # the dominant GEMM's own FLOPs: QKV 2 tok C 3C, projection 2 tok C C, per layer
        per = sum((2 * ly.B * ly.T * ly.H * ly.W * ly.C * (3 * ly.C if dom == "qkv_gemm" else ly.C))
                  for ly in layers)
        dom_work, unit, bound = per * args.steps, "TFLOP/s", "tensor"
        achieved = dom_work / (dom_ms / 1e3) / 1e12
        peak = float(peaks["bf16_tflops"])
        traffic_kernel = "gemm_kernel" if dom == "qkv_gemm" else "proj_kernel"
    tr = traffic_record(traffic_kernel, args.workload)
    avg_us = 1e3 * dom_ms / max(1, dom_launches)
    roofline = {
        "kernel": dom, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
        "frac": achieved / peak, "peak_source": f"{peak_src} bf16 dense (burst)",
        "avg_launch_us": avg_us, "launches": dom_launches,
        "traffic": tr["bytes_per_launch"] if tr else None,
        "units_per_launch": "windows x heads of one chunk; FLOPs 4*windows*N^2*C per layer",
    }
    if dom == "attention":
        # the exponentials' own floor on the MUFU (16 ex2 / clock / SM) at the clock seen
        # during the timed region, beside the tensor roofline
        mhz = clocks.get("sm_mhz") or clocks.get("sm_max_mhz") or 1965.0
        exps_launch = work["exps"] / len(layers)
        roofline["exp_bound_us"] = exp_bound_us(exps_launch, mhz)
        roofline["exp_bound_frac"] = roofline["exp_bound_us"] / avg_us
        roofline["exp_bound_note"] = (f"{exps_launch:.4g} exponentials per launch (every pair, masked ones "
                                      f"included) / (148 SMs x 16 per clock x {mhz:.0f} MHz)")
    kernel_ms = {k: v[0] / args.steps for k, v in prof.items() if v[1]}
    step_flops_time = work["flops"] / (float(peaks["bf16_tflops"]) * 1e12)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": nranks, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * max_s / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(wl),
        "tflops": tflops,
        "tflops_frac_of_peak": tflops / nranks / float(peaks["bf16_tflops"]),
        "step_roofline_us": 1e6 * max(step_flops_time, work["bytes"] / (float(peaks["hbm_gbs"]) * 1e9)),
        "roofline": roofline,
        "kernel_ms_per_step": kernel_ms,
        "step_ms": step_stats,
        "warm_l2": {"value": warm_tokens / warm_max_s, "ms_per_step": 1e3 * warm_max_s / n_warm, "steps": n_warm,
                    "note": "no L2 flush between steps"},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if world == 1 and not args.no_cpu_baseline:
        s = oracle_sample(wl, args.cpu_sample_s)
        line["cpu_baseline"] = {
            "value": s["tokens"] / s["seconds"], "unit": "tokens/s", "cores": s["cores"], "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"{s['windows_per_layer']} evenly spaced whole windows of each layer of the pair "
                      f"({s['tokens']} layer-tokens, {s['seconds']:.1f} s), double precision",
        }
    print(json.dumps(line), flush=True)
    replicas.shutdown()
    return 0


def run_block(args):
    """``--block``: the attention half of the blocks on the same workload, out = x +
    layer(LN(x)) per layer, through the fused entry (vswin_block_msa_forward) and,
    for comparison, unfused (torch layer_norm, vswin_wmsa_forward, torch add). One
    GPU; prints its own JSON line."""
    from shifted_window_attention_sw_b200 import build as build_mod
    from shifted_window_attention_sw_b200 import vswin
    from shifted_window_attention_sw_b200.inputs import make_block_inputs

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    build_mod.build()
    vswin.lib()
    wl = WORKLOADS[args.workload]
    layers = wl.layers
    base = 1000 * wl.index
    bins = [make_block_inputs(ly.shape, ly.heads, ly.window, wl.dtype, "baseline", seed=base + ly.seed_offset,
                              x_seed=base).to(device) for ly in layers]
    outs = [torch.empty_like(b.layer.x) for b in bins]
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    eps = 1e-5

    def fused():
        for ly, b, o in zip(layers, bins, outs):
            li = b.layer
            vswin.block_msa_forward(li.x, ly.window, ly.shift, b.gamma, b.beta, eps, li.Wqkv, li.bqkv, li.Wproj,
                                    li.bproj, li.table, ly.heads, out=o, stream=stream)

    def unfused():
        for ly, b, o in zip(layers, bins, outs):
            li = b.layer
            y = torch.nn.functional.layer_norm(li.x, (ly.C,), b.gamma, b.beta, eps)
            vswin.wmsa_forward(y, ly.window, ly.shift, li.Wqkv, li.bqkv, li.Wproj, li.bproj, li.table, ly.heads,
                               out=o, stream=stream)
            o.add_(li.x)

    def timed(fn, profile):
        for _ in range(args.warmup):
            flush.zero_()
            fn()
        torch.cuda.synchronize(device)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        launches0 = vswin.launch_count()
        if profile:
            vswin.profile_enable(True)
        sampler = ClockSampler(device)
        sampler.start()
        for k in range(args.steps):
            flush.zero_()
            evs[k][0].record(stream)
            fn()
            evs[k][1].record(stream)
        torch.cuda.synchronize(device)
        clocks = sampler.stop()
        prof = None
        if profile:
            vswin.profile_enable(False)
            prof = vswin.profile_collect()
        if vswin.poll_error(stream) != vswin.OK:
            raise RuntimeError("kernel error in the timed region: " + vswin.last_error())
        ms = [a.elapsed_time(b) for a, b in evs]
        return sum(ms) / len(ms), prof, vswin.launch_count() - launches0, clocks

    f_ms, prof, launches, clocks = timed(fused, True)
    u_ms, _, _, u_clocks = timed(unfused, False)
    tokens = step_work(wl)["tokens"]
    cfg = workload_config(wl)
    cfg["ln_eps"] = eps
    line = {
        "metric": "block attention-half tokens/s (LN + (S)W-MSA + residual), " + wl.name,
        "value": tokens / (f_ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": f_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
        "api": "vswin_block_msa_forward",
        "kernel_ms_per_step": {k: v[0] / args.steps for k, v in prof.items() if v[1]},
        "gpu_launches": int(launches),
        "unfused": {"ms_per_step": u_ms, "value": tokens / (u_ms / 1e3),
                    "what": "torch layer_norm + vswin_wmsa_forward + torch add_", "clocks": u_clocks},
        "fused_speedup": u_ms / f_ms,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_backward(args):
    """``--backward``: the fp32 backward (vswin_wmsa_backward_f32: forward recompute plus
    every gradient) of each layer of the workload, on fp32 inputs of the same shapes. One
    GPU; prints its own JSON line. The path is plain FP32 arithmetic, so the roofline is
    the FP32 ALU peak: 148 SMs x 128 FP32 lanes x 2 FLOP x 1.965 GHz = 74.4 TFLOP/s."""
    from shifted_window_attention_sw_b200 import build as build_mod
    from shifted_window_attention_sw_b200 import vswin
    from shifted_window_attention_sw_b200.inputs import make_layer_inputs

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    build_mod.build()
    vswin.lib()
    wl = WORKLOADS[args.workload]
    layers = wl.layers
    base = 1000 * wl.index
    ins = [make_layer_inputs(ly.shape, ly.heads, ly.window, "f32", "baseline", seed=base + ly.seed_offset,
                             x_seed=base).to(device) for ly in layers]
    dys = [torch.randn(*ly.shape, generator=torch.Generator().manual_seed(base + 77 + k)).to(device)
           for k, ly in enumerate(layers)]
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        for ly, i, dy in zip(layers, ins, dys):
            vswin.wmsa_backward_f32(i.x, ly.window, ly.shift, i.Wqkv, i.bqkv, i.Wproj, i.bproj, i.table, ly.heads,
                                    dy, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    launches0 = vswin.launch_count()
    sampler = ClockSampler(device)
    sampler.start()
    for k in range(args.steps):
        flush.zero_()
        evs[k][0].record(stream)
        step()
        evs[k][1].record(stream)
    torch.cuda.synchronize(device)
    clocks = sampler.stop()
    if vswin.poll_error(stream) != vswin.OK:
        raise RuntimeError("kernel error in the timed region: " + vswin.last_error())
    ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    # FLOPs of the kernels as built, per layer (rows = window slots, masked pairs
    # included): qkv recompute 2 rows C 3C; dO 2 rows C^2; per window, the query
    # pass 10 N^2 C (scores twice, O, dP, dq) and the key pass 8 N^2 C (scores,
    # dP, dk, dv); dx 2 rows 3C C; dWqkv 2 rows C 3C; dWproj 2 rows C^2
    flops = 0
    for ly in layers:
        g = layer_work(ly.B, ly.T, ly.H, ly.W, ly.C, ly.heads, ly.window, ly.shift, 4)
        win, N = g["windows"], g["N"]
        rows = win * N
        C = ly.C
        flops += 2 * rows * C * 3 * C * 3 + 2 * rows * C * C * 2 + (10 + 8) * win * N * N * C
    tokens = step_work(wl)["tokens"]
    achieved = flops / (ms / 1e3) / 1e12
    peak = 148 * 128 * 2 * 1.965e9 / 1e12
    line = {
        "metric": "fp32 layer backward tokens/s (forward recompute + all gradients), " + wl.name,
        "value": tokens / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": workload_config(wl),
        "api": "vswin_wmsa_backward_f32",
        "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "peak_source": "148 SMs x 128 FP32 lanes x 2 x 1.965 GHz",
                     "flops_per_step": flops},
        "gpu_launches": int(vswin.launch_count() - launches0),
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0



def run_backward_bf16(args):
    """``--backward-bf16``: the bf16 tensor-core backward (vswin_wmsa_backward: the forward's
    first three steps recomputed with the softmax statistics, dO, the attention gradients
    on tcgen05, dX and the fp32 weight gradients) of each layer of the workload. One GPU;
    prints its own JSON line with the attention-gradient kernel's roofline against the
    bf16 tensor peak and its exponential (MUFU) bound."""
    from shifted_window_attention_sw_b200 import build as build_mod
    from shifted_window_attention_sw_b200 import vswin
    from shifted_window_attention_sw_b200.inputs import make_layer_inputs

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    build_mod.build()
    vswin.lib()
    wl = WORKLOADS[args.workload]
    layers = wl.layers
    base = 1000 * wl.index
    ins = [make_layer_inputs(ly.shape, ly.heads, ly.window, "bf16", "baseline", seed=base + ly.seed_offset,
                             x_seed=base).to(device) for ly in layers]
    dys = [torch.randn(*ly.shape, generator=torch.Generator().manual_seed(base + 77 + k)).bfloat16().to(device)
           for k, ly in enumerate(layers)]
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        for ly, i, dy in zip(layers, ins, dys):
            vswin.wmsa_backward(i.x, ly.window, ly.shift, i.Wqkv, i.bqkv, i.Wproj, i.bproj, i.table, ly.heads,
                                dy, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    launches0 = vswin.launch_count()
    vswin.profile_enable(True)
    sampler = ClockSampler(device)
    sampler.start()
    for k in range(args.steps):
        flush.zero_()
        evs[k][0].record(stream)
        step()
        evs[k][1].record(stream)
    torch.cuda.synchronize(device)
    clocks = sampler.stop()
    vswin.profile_enable(False)
    prof = vswin.profile_collect()
    if vswin.poll_error(stream) != vswin.OK:
        raise RuntimeError("kernel error in the timed region: " + vswin.last_error())
    ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    # tensor-core FLOPs as built, per layer (rows = window slots, masked pairs
    # included): attention gradients 10 N^2 d per (window, head) (S^T, dP^T, dV, dK,
    # dQ), the recomputed attention 4 N^2 d, and the products qkv 2 rows C 3C, dO
    # 2 rows C^2, dx 2 rows 3C C; the two weight-gradient sums (2 rows C 3C + 2 rows
    # C^2) run on the FP32 pipes
    attn_flops = tc_flops = simt_flops = exps = 0
    for ly in layers:
        g = layer_work(ly.B, ly.T, ly.H, ly.W, ly.C, ly.heads, ly.window, ly.shift, 4)
        win, N = g["windows"], g["N"]
        rows = win * N
        C = ly.C
        attn_flops += 10 * win * N * N * C
        tc_flops += 14 * win * N * N * C + 2 * rows * C * 3 * C * 2 + 2 * rows * C * C
        simt_flops += 2 * rows * C * 3 * C + 2 * rows * C * C
        exps += win * N * N * ly.heads
    tokens = step_work(wl)["tokens"]
    line = {
        "metric": "bf16 layer backward tokens/s (forward recompute + all gradients), " + wl.name,
        "value": tokens / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_config(wl),
        "api": "vswin_wmsa_backward",
        "tensor_flops_per_step": tc_flops, "fp32_flops_per_step": simt_flops,
        "kernel_ms_per_step": {k: v[0] / args.steps for k, v in prof.items() if v[1]},
        "gpu_launches": int(vswin.launch_count() - launches0),
        "clocks": clocks,
    }
    a_ms, a_n = prof["attention_bwd"]
    if a_n:
        avg_us = a_ms / a_n * 1e3
        per_launch = attn_flops * args.steps / a_n  # one launch per layer and chunk
        achieved = per_launch / (avg_us / 1e6) / 1e12
        peaks, psrc = load_peaks()
        peak, src = float(peaks["bf16_tflops"]), f"{psrc} bf16 dense (burst)"
        exp_us = exps * args.steps / a_n / (148 * 16 * 1.965e9) * 1e6
        line["roofline"] = {
            "kernel": "bwd_attn_kernel", "bound": "tensor", "achieved": achieved, "peak": peak,
            "unit": "TFLOP/s", "frac": achieved / peak, "peak_source": src, "avg_launch_us": avg_us,
            "launches": a_n, "traffic": None,
            "units_per_launch": "windows x heads of one chunk; FLOPs 10*windows*N^2*C (S^T, dP^T, dV, dK, dQ)",
            "exp_bound_us": exp_us, "exp_bound_frac": exp_us / avg_us,
            "exp_bound_note": "one exponential per (query, key, head), masked pairs included, at 16 per clock per SM"}
    print(json.dumps(line), flush=True)
    return 0

def run_mlp(args):
    """``--mlp``: the fused MLP half (vswin_mlp_forward, hidden 4C) on each layer's token
    tensor; ``--block-full``: whole blocks, the attention half (vswin_block_msa_forward)
    then the MLP half, per layer of the workload. One GPU; prints its own JSON line."""
    from shifted_window_attention_sw_b200 import build as build_mod
    from shifted_window_attention_sw_b200 import vswin
    from shifted_window_attention_sw_b200.inputs import make_block_inputs, make_mlp_inputs

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    build_mod.build()
    vswin.lib()
    wl = WORKLOADS[args.workload]
    layers = wl.layers
    base = 1000 * wl.index
    mlps = [make_mlp_inputs(ly.shape, 4 * ly.C, wl.dtype, "baseline", seed=base + ly.seed_offset).to(device)
            for ly in layers]
    blocks = ([make_block_inputs(ly.shape, ly.heads, ly.window, wl.dtype, "baseline", seed=base + ly.seed_offset,
                                 x_seed=base).to(device) for ly in layers] if args.block_full else None)
    outs = [torch.empty_like(m.x) for m in mlps]
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    eps = 1e-5

    def step():
        for k, (ly, m, o) in enumerate(zip(layers, mlps, outs)):
            src = m.x
            if blocks is not None:
                b = blocks[k]
                li = b.layer
                vswin.block_msa_forward(li.x, ly.window, ly.shift, b.gamma, b.beta, eps, li.Wqkv, li.bqkv,
                                        li.Wproj, li.bproj, li.table, ly.heads, out=o, stream=stream)
                src = o
            vswin.mlp_forward(src, m.gamma, m.beta, eps, m.W1, m.b1, m.W2, m.b2, out=o, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(device)
    if vswin.poll_error(stream) != vswin.OK:
        raise RuntimeError("kernel error during warm-up: " + vswin.last_error())
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    launches0 = vswin.launch_count()
    vswin.profile_enable(True)
    sampler = ClockSampler(device)
    sampler.start()
    for k in range(args.steps):
        flush.zero_()
        evs[k][0].record(stream)
        step()
        evs[k][1].record(stream)
    torch.cuda.synchronize(device)
    clocks = sampler.stop()
    vswin.profile_enable(False)
    prof = vswin.profile_collect()
    if vswin.poll_error(stream) != vswin.OK:
        raise RuntimeError("kernel error in the timed region: " + vswin.last_error())
    ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    peaks, peak_src = load_peaks()
    tokens = sum(ly.B * ly.T * ly.H * ly.W for ly in layers)
    mlp_flops = sum(2 * 2 * ly.B * ly.T * ly.H * ly.W * ly.C * 4 * ly.C for ly in layers)
    mlp_bytes = sum(2 * 2 * ly.B * ly.T * ly.H * ly.W * ly.C + 2 * 2 * 4 * ly.C * ly.C for ly in layers)
    mlp_ms, mlp_n = prof["mlp"]
    mlp_us = 1e3 * mlp_ms / max(1, mlp_n)
    achieved = mlp_flops / len(layers) / (mlp_us / 1e6) / 1e12
    peak = float(peaks["bf16_tflops"])
    gelus = sum(ly.B * ly.T * ly.H * ly.W * 4 * ly.C for ly in layers) / len(layers)
    mhz = clocks.get("sm_mhz") or clocks.get("sm_max_mhz") or 1965.0
    what = "whole block (attention half + MLP half)" if args.block_full else "MLP half (LN, fc1, GELU, fc2, residual)"
    line = {
        "metric": f"{what} tokens/s, {wl.name}", "value": tokens / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(wl), hidden="4C", ln_eps=eps),
        "api": "vswin_block_msa_forward + vswin_mlp_forward" if args.block_full else "vswin_mlp_forward",
        "kernel_ms_per_step": {k: v[0] / args.steps for k, v in prof.items() if v[1]},
        "mlp_roofline": {"kernel": "mlp_kernel", "bound": "tensor", "achieved": achieved, "peak": peak,
                         "traffic": (traffic_record("mlp_kernel", args.workload) or {}).get("bytes_per_launch"),
                         "unit": "TFLOP/s", "frac": achieved / peak, "peak_source": f"{peak_src} bf16 dense (burst)",
                         "avg_launch_us": mlp_us, "launches": mlp_n,
                         "hbm_floor_us": mlp_bytes / len(layers) / (float(peaks["hbm_gbs"]) * 1e9) * 1e6,
                         "tanh_bound_us": gelus / (SMS * MUFU_EX2_PER_CLK_SM * mhz * 1e6) * 1e6,
                         "units_per_launch": "one layer's tokens; FLOPs 4*tok*C*hidden, hidden = 4C"},
        "gpu_launches": int(vswin.launch_count() - launches0),
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_merge(args):
    """``--merge``: patch merging (vswin_patch_merge_forward) of each layer's token tensor
    of the workload, the step between Video Swin stages. One GPU; prints its own JSON line."""
    from shifted_window_attention_sw_b200 import build as build_mod
    from shifted_window_attention_sw_b200 import vswin
    from shifted_window_attention_sw_b200.inputs import make_merge_inputs

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    build_mod.build()
    vswin.lib()
    wl = WORKLOADS[args.workload]
    layers = wl.layers
    base = 1000 * wl.index
    ins = [make_merge_inputs(ly.shape, wl.dtype, "baseline", seed=base + ly.seed_offset).to(device) for ly in layers]
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    eps = 1e-5

    def step():
        for m in ins:
            vswin.patch_merge_forward(m.x, m.gamma, m.beta, eps, m.Wr, m.br, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    launches0 = vswin.launch_count()
    vswin.profile_enable(True)
    sampler = ClockSampler(device)
    sampler.start()
    for k in range(args.steps):
        flush.zero_()
        evs[k][0].record(stream)
        step()
        evs[k][1].record(stream)
    torch.cuda.synchronize(device)
    clocks = sampler.stop()
    vswin.profile_enable(False)
    prof = vswin.profile_collect()
    if vswin.poll_error(stream) != vswin.OK:
        raise RuntimeError("kernel error in the timed region: " + vswin.last_error())
    ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    peaks, peak_src = load_peaks()
    tokens = sum(ly.B * ly.T * ly.H * ly.W for ly in layers)
    merged = sum(ly.B * ly.T * ((ly.H + 1) // 2) * ((ly.W + 1) // 2) for ly in layers)
    flops = sum(2 * ly.B * ly.T * ((ly.H + 1) // 2) * ((ly.W + 1) // 2) * 4 * ly.C * 2 * ly.C for ly in layers)
    byts = sum(2 * ly.B * ly.T * ly.H * ly.W * ly.C + 2 * ly.B * ly.T * ((ly.H + 1) // 2) * ((ly.W + 1) // 2) * 2 * ly.C
               for ly in layers)
    k_ms, k_n = prof["mlp"]  # the merge GEMM is timed in the MLP kind
    k_us = 1e3 * k_ms / max(1, k_n)
    line = {
        "metric": f"patch merging input tokens/s, {wl.name}", "value": tokens / (ms / 1e3), "unit": "tokens/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(wl), merged_tokens=merged, ln_eps=eps), "api": "vswin_patch_merge_forward",
        "kernel_ms_per_step": {k: v[0] / args.steps for k, v in prof.items() if v[1]},
        "merge_roofline": {"kernel": "pm_ws_kernel", "bound": "hbm", "achieved": byts / len(layers) / (k_us / 1e6) / 1e9,
                           "traffic": (traffic_record("merge_kernel", wl.name) or {}).get("bytes_per_launch"),
                           "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                           "frac": byts / len(layers) / (k_us / 1e6) / 1e9 / float(peaks["hbm_gbs"]),
                           "peak_source": f"{peak_src} HBM copy", "avg_launch_us": k_us,
                           "tflops": flops / len(layers) / (k_us / 1e6) / 1e12,
                           "units_per_launch": "one layer's tokens; bytes = x read + merged output written"},
        "gpu_launches": int(vswin.launch_count() - launches0),
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["vswin", "reference"], default="vswin")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=HEADLINE)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-s", type=float, default=20.0)
    ap.add_argument("--block", action="store_true",
                    help="time the blocks' attention half (LN, layer, residual), fused and unfused, on one GPU")
    ap.add_argument("--backward-bf16", action="store_true",
                    help="time the bf16 tensor-core backward of each layer of the workload on one GPU")
    ap.add_argument("--backward", action="store_true",
                    help="time the fp32 backward of each layer of the workload on one GPU")
    ap.add_argument("--mlp", action="store_true",
                    help="time the fused MLP half of a block (hidden 4C) on each layer's tokens, one GPU")
    ap.add_argument("--merge", action="store_true",
                    help="time patch merging (2x2 neighbours, LN over 4C, 4C -> 2C) of each layer's tokens, one GPU")
    ap.add_argument("--block-full", action="store_true",
                    help="time whole blocks (attention half then MLP half) on the workload's layers, one GPU")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "0"))
    if args.gpus > 1 and world == 0 and not (args.block or args.backward or args.backward_bf16 or args.mlp or args.block_full or args.merge):
        # one process per GPU: relaunch this command under torchrun
        import socket

        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
               "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__),
               *(argv if argv is not None else sys.argv[1:])]
        os.execv(sys.executable, cmd)
    if world and world != args.gpus:
        ap.error(f"--gpus {args.gpus} does not match WORLD_SIZE={world}")
    if args.impl == "reference":
        return run_reference(args)
    if args.block:
        return run_block(args)
    if args.backward:
        return run_backward(args)
    if args.backward_bf16:
        return run_backward_bf16(args)
    if args.mlp or args.block_full:
        return run_mlp(args)
    if args.merge:
        return run_merge(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
