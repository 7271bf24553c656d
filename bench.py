#!/usr/bin/env python
"""Throughput of the Nemotron-H MoE FFN layer forward on B200 (tokens/s).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--tokens T] [--impl ours|reference]

One step = one full forward of the layer (norm, router, top-k, sort, experts,
shared expert, reduce, residual) over one batch of T synthetic tokens with
inputs resident in HBM.  The default workload is the decode configuration at
T=1 (H=2688, E=128, top_k=6, moe_inter=1856, shared 3712, BF16 weights).
L2 is flushed (256 MB write, then 256 MB read) between timed steps; every step restores the
same input tokens, so routing and work are identical across steps.

Multi-GPU (torchrun, one rank per GPU): tokens are independent, so every
rank runs its own replica on its own batch with no data-path collective
(weak scaling); NCCL is used only for the barrier and the max-over-ranks
time.  Rank 0 prints one JSON line.

--impl reference times the float64 CPU oracle on the host cores instead, on
a bounded sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "MoE-layer tokens/sec"
UNIT = "tokens/s"
DEFAULT_TOKENS = {"tiny": 16, "decode": 1, "prefill": 1024, "latent": 4096, "skew_fp8": 8192}


# ------------------------------------------------------------------ peaks ---

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ------------------------------------------------------- work per kernel ---

def stage_model(s, T, path, U, router_split=False):
    """Algorithmic bytes / flops of every kernel the chosen path launches.

    U = distinct routed experts of the step (weights touched once each).
    Weight bytes use the storage width (2 for BF16, 1 for FP8 + scales).
    Returns a list of (name, bytes, flops, fp8_flops) in launch order:
    `flops` counts all of a kernel's multiply-adds (x2), `fp8_flops` the part
    of them that runs on E4M3 operands (the routed experts when their weights
    are FP8; the gate, the shared expert and fc1/fc2 are BF16).
    """
    H, E, k, I, S, L = s.H, s.E, s.k, s.I, s.S, s.L
    D = s.D
    R = T * k
    wb = 1 if s.expert_fp8 else 2
    up_w = U * I * D * wb + (U * I * 4 if s.expert_fp8 else 0)
    down_w = U * D * I * wb + (U * D * 4 if s.expert_fp8 else 0)
    f8 = 1 if s.expert_fp8 else 0
    if path == "decode":
        # one launch: the whole forward (its up outputs and partial sums stay
        # in L2 and are not counted)
        nb, fl, f8f = step_work(s, T, U)
        return [("decode_fused", nb, fl, f8f)]
    # RMSNorm: x in, residual and the bf16 normed rows out, r per token (and
    # the E4M3 copy with FP8 experts)
    st = [("rmsnorm", T * H * 2 * 3 + T * 4 + (T * H + T * 4 if s.expert_fp8 else 0), 0, 0)]
    # With split K (few token tiles) the router GEMM stores partial logits
    # and a second kernel sums them and selects; its algorithmic bytes are
    # the routing table it writes (the partials are the split's overhead).
    sel = "" if router_split else "_topk"
    # the router reads the raw rows x (once; its second pass along K hits L2)
    # and the gate with the norm weight folded in, as BF16 hi and lo halves
    if L:
        st.append((f"router_gemm{sel}+fc1", E * 2 * H * 2 + T * H * 2 + L * H * 2 + T * H * 2
                   + T * L * 2, 2 * T * E * H + 2 * T * H * L, 0))
    else:
        st.append((f"router_gemm{sel}", E * 2 * H * 2 + T * H * 2 + (0 if router_split else R * 8),
                   2 * T * E * H, 0))
    if router_split:
        st.append(("router_reduce_topk", R * 8, 0, 0))
    st += [
        ("sort", R * 4 * 3 + (E + 1) * 4, 0, 0),
        # each token row is read once from HBM (its k copies come from L2)
        # and written once per routed slot
        ("gather", T * D * wb + R * D * wb + R * 4, 0, 0),
        ("grouped_up_gemm", up_w + S * H * 2 + R * D * wb + T * H * 2 + R * I * 2 + T * S * 2,
         2 * R * D * I + 2 * T * H * S, f8 * 2 * R * D * I),
    ]
    if s.expert_fp8:
        st.append(("quantize_rows", R * I * 2 + R * I + R * 8, 0, 0))
    st += [
        ("grouped_down_gemm", down_w + H * S * 2 + R * I * wb + T * S * 2 + R * D * 2 + T * H * 4,
         2 * R * I * D + 2 * T * S * H, f8 * 2 * R * I * D),
    ]
    if L:
        st += [("latent_reduce", R * L * 2 + T * L * 2, 0, 0),
               ("fc2_gemm_blend", H * L * 2 + T * L * 2 + T * H * (4 + 2 + 2), 2 * T * L * H, 0)]
    else:
        st.append(("combine", R * D * 2 + T * H * 4 + T * H * 2 * 2, 0, 0))
    return st


def step_work(s, T, U):
    """What one forward must move and compute at least, whatever its kernels:
    the gate, the U touched experts' weights, the shared expert, fc1/fc2, the
    norm weight, and the token rows (hidden in, hidden out, residual out).
    Returns (bytes, flops, fp8_flops)."""
    H, E, k, I, S, L, D = s.H, s.E, s.k, s.I, s.S, s.L, s.D
    R = T * k
    wb = 1 if s.expert_fp8 else 2
    scales = U * (I + D) * 4 if s.expert_fp8 else 0
    nbytes = (E * H * 2 + U * 2 * D * I * wb + scales + 2 * H * S * 2 + 2 * H * L * 2 + H * 2
              + 3 * T * H * 2)
    routed = 4 * R * D * I
    flops = 2 * T * H * E + routed + 4 * T * H * S + 4 * T * H * L
    return nbytes, flops, (routed if s.expert_fp8 else 0)


def roofline_of(name, nbytes, flops, ms, peaks, fp8_flops=0):
    """The binding bound of `nbytes` and `flops` done in `ms`: HBM time at
    the measured copy bandwidth, tensor time with the BF16 flops at the
    measured BF16 peak and the FP8 flops at twice it (the nominal FP8/BF16
    ratio), each class at its own rate.  frac = bound time / measured time."""
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    bf = peaks["bf16_tflops"] * 1e12
    t_tc = (flops - fp8_flops) / bf + fp8_flops / (2.0 * bf)
    if t_tc > t_hbm:
        ach = flops / (ms * 1e-3) / 1e12
        peak = flops / t_tc / 1e12  # BF16 peak, 2x for FP8, mixed by flops
        return {"bound": "tensor", "achieved": round(ach, 2), "peak": round(peak, 1),
                "unit": "TFLOP/s", "frac": round(t_tc / (ms * 1e-3), 4)}
    ach = nbytes / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(ach / peaks["hbm_gbs"], 4)}


def kernel_traffic(name, workload):
    """dram bytes per launch of kernel stage `name` on `workload` ("prefill
    T=1024") from the committed ncu summary, or None when there is no capture
    of that pair or the kernel source or launch configuration has changed
    since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    rec = d.get("kernels", {}).get(f"{name}@{workload}")
    if not rec:
        return None
    return rec["dram_bytes_per_launch"] if sources_hash(rec["sources"]) == rec.get(
        "sources_sha256_16") else None


def sources_hash(paths):
    """sha256 prefix over the kernel source and the launch configuration that
    determine a kernel's traffic (files relative to the repository root)."""
    h = hashlib.sha256()
    try:
        for rel in paths:
            with open(os.path.join(ROOT, rel), "rb") as f:
                h.update(f.read())
    except OSError:
        return None
    return h.hexdigest()[:16]


# ------------------------------------------------------------ multi-rank ---

def max_over_ranks(ms, world, device):
    """The job's time for a quantity every rank measured on its own device:
    the slowest rank's (all-reduce MAX; with the barriers around the timed
    region this is the only collective, the replicas share no data)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world, T, steps, ms):
    """Whole-job throughput: every rank processes its own T tokens per step."""
    return world * T * steps / (ms * 1e-3)


# --------------------------------------------------------------- clocks ---

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index, interval=0.002):
        self.samples = []
        self.reasons = 0
        self.interval = interval
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.interval)

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": "nvml unavailable"}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples), "source": "nvml in-process"}


# --------------------------------------------------------- CPU baseline ---

def cpu_baseline(inp, T, target_s=10.0):
    """The float64 oracle as it stands, on host threads, over a bounded
    sample of the same workload (same weights, more tokens)."""
    import oracle
    s = inp.shape
    threads = oracle.default_threads()
    orc = oracle.Oracle(inp)
    probe = make_inputs(s, T=max(threads, 1), experts=False).hidden
    t0 = time.perf_counter()
    orc.forward(probe, nthreads=threads)
    per_tok = (time.perf_counter() - t0) / probe.shape[0]
    n = int(min(4096, max(threads, target_s / max(per_tok, 1e-9))))
    n = max(threads, (n // threads) * threads)
    sample = make_inputs(s, T=n, experts=False).hidden
    t0 = time.perf_counter()
    orc.forward(sample, nthreads=threads)
    dt = time.perf_counter() - t0
    return {"value": round(n / dt, 3), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n} tokens of the {s.name} workload (same weights), float64 C++ oracle "
                      f"threaded over tokens, {dt:.1f} s"}


# ------------------------------------------------------------ reference ---

def run_reference(args, shape, T, rank, world):
    if rank != 0:
        return
    import oracle
    inp = make_inputs(shape, T=T)
    orc = oracle.Oracle(inp)
    threads = oracle.default_threads()
    # per-step sample: as many of the T tokens as keep the whole run short
    t0 = time.perf_counter()
    orc.forward(inp.hidden[:1], nthreads=threads)
    per_tok = time.perf_counter() - t0
    budget = 150.0
    n = int(max(1, min(T, budget / max(per_tok * (args.steps + args.warmup), 1e-9) * threads)))
    h = inp.hidden[:n]
    for _ in range(args.warmup):
        orc.forward(h, nthreads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        orc.forward(h, nthreads=threads)
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(shape, T, "oracle"),
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": threads,
                             "kind": "oracle",
                             "sample": f"{n} of the {T} tokens per step, float64 C++ oracle, "
                                       f"{threads} threads"},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(s, T, path):
    w = "FP8 E4M3 experts" if s.expert_fp8 else "BF16"
    lat = f", latent={s.L}" if s.L else ""
    return {"workload": f"{s.name} T={T} (H={s.H}, E={s.E}, top_k={s.k}, moe_inter={s.I}, "
                        f"shared={s.S}{lat}, {w}, rsf={s.rsf})",
            "tokens_per_step": T, "path": path, "l2": "flushed between timed steps (256 MB write + 256 MB read)"}


# ------------------------------------------------------------------ ours ---

# Workloads measured after the headline one in the same run (N = 1), each at
# the token count its configuration names; decode also at T = 8, the largest
# batch of the decode path.
SUB_WORKLOADS = (("decode", 8), ("tiny", 16), ("prefill", 1024), ("latent", 4096),
                 ("skew_fp8", 8192), ("skew_fp8", 1))  # (the last: its FP8 layer at decode)

STAGE_NOTE = ("per-kernel times come from a second CUDA graph with events recorded between "
              "the kernels; those events break the programmatic-dependent-launch overlap, so "
              "the stage times sum to more than ms_per_step and each stage's frac is a lower bound")


class L2Flush:
    """Writes 256 MB (evicting everything), then reads another 256 MB so L2
    holds clean lines and the next step pays no write-backs."""

    def __init__(self):
        import torch
        self.w = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
        self.r = torch.zeros(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
        self.out = torch.empty((), dtype=torch.float32, device="cuda")

    def __call__(self):
        import torch
        self.w.zero_()
        torch.amax(self.r, dim=0, out=self.out)


def measure(inp, T, args, world, flush, peaks, *, e2e=True):
    """Time `args.steps` forwards of T tokens of `inp` after `args.warmup`
    untimed ones (CUDA-graph replay unless --eager, L2 flushed between
    steps), on the device with CUDA events; the time is the max over ranks.
    Returns the workload's record (throughput, roofline, stages, clocks,
    end-to-end through the host-buffer entry point)."""
    import torch
    import torch.distributed as dist

    import mixture_experts_ffn_rmsnorm_b200 as moe

    fpath = {"auto": moe.PATH_AUTO, "decode": moe.PATH_DECODE,
             "prefill": moe.PATH_PREFILL}[getattr(args, "path", "auto")]

    shape = inp.shape
    layer = moe.MoELayer.from_inputs(inp, max_tokens=T)
    hbits = inp.hidden[:T]
    pristine = torch.from_numpy(hbits.view(np.int16).copy()).cuda()
    hid = torch.empty_like(pristine)
    res = torch.empty_like(pristine)
    stream = torch.cuda.current_stream()

    # one untimed step to learn the launch count, the path and the routing
    hid.copy_(pristine)
    layer.forward(hid, res, path=fpath)
    torch.cuda.synchronize()
    nl = layer.last_launch_count()
    path = "decode" if layer.last_path_decode() else "prefill"
    idx = torch.empty((T, shape.k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, shape.k), dtype=torch.float32, device="cuda")
    layer.copy_routing(idx, wts)
    U = int(torch.unique(idx).numel())

    def make_events(n):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in ev:
            e.record(stream)
        return ev

    for _ in range(args.warmup):
        flush()
        hid.copy_(pristine)
        layer.forward(hid, res, path=fpath)
    torch.cuda.synchronize()

    # The step: one replay of a CUDA graph of the forward (what a serving loop
    # does for a layer), or an eager call with --eager.  A second graph with
    # CUDA events captured between the kernels gives the per-kernel times.
    graph = prof_graph = None
    prof_events = make_events(nl + 1)
    if not args.eager:
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            layer.forward(hid, res, path=fpath, stream=side)
        prof_graph = torch.cuda.CUDAGraph()
        layer.set_stage_events(prof_events)
        with torch.cuda.graph(prof_graph, stream=side):
            layer.forward(hid, res, path=fpath, stream=side)
        layer.set_stage_events(None)
        stream.wait_stream(side)
        for _ in range(args.warmup):
            flush()
            hid.copy_(pristine)
            graph.replay()
        torch.cuda.synchronize()

    e_start = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_end = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        for i in range(args.steps):
            flush()
            hid.copy_(pristine)
            e_start[i].record(stream)
            if graph is not None:
                graph.replay()
            else:
                layer.forward(hid, res, path=fpath)
            e_end[i].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
    step_ms = np.array([a.elapsed_time(b) for a, b in zip(e_start, e_end)])
    total_ms = max_over_ranks(float(step_ms.sum()), world, "cuda")
    value = job_tokens_per_s(world, T, args.steps, total_ms)
    ms_step = total_ms / args.steps

    # per-kernel device times: events recorded between the launches
    n_prof = min(args.steps, 50)
    stage_ms = np.zeros((n_prof, nl))
    if prof_graph is None:
        layer.set_stage_events(prof_events)
    for i in range(n_prof):
        flush()
        hid.copy_(pristine)
        if prof_graph is not None:
            prof_graph.replay()
        else:
            layer.forward(hid, res, path=fpath)
        torch.cuda.synchronize()
        stage_ms[i] = [prof_events[j].elapsed_time(prof_events[j + 1]) for j in range(nl)]
    layer.set_stage_events(None)

    e2e_rec = None
    # (the host-buffer entry point chooses the path itself: no end-to-end
    # figure for a forced path)
    if e2e and getattr(args, "path", "auto") == "auto":
        # end to end through the host-buffer entry point (pinned host memory)
        h_host = torch.from_numpy(hbits.view(np.int16).copy()).pin_memory()
        e0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        e1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        src = hbits.view(np.int16)
        for i in range(args.steps):
            h_host.numpy()[...] = src
            flush()
            e0[i].record(stream)
            layer.forward_host(h_host)
            e1[i].record(stream)
            stream.synchronize()
        e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(e0, e1)), world, "cuda")
        e2e_rec = {"value": round(job_tokens_per_s(world, T, args.steps, e2e_ms), 2),
                   "unit": UNIT, "h2d_bytes_per_step": T * shape.H * 2,
                   "d2h_bytes_per_step": T * shape.H * 2}
    layer.close()

    model = stage_model(shape, T, path, U)
    if path == "prefill" and len(model) + 1 == nl:
        model = stage_model(shape, T, path, U, router_split=True)
    if len(model) != nl:  # keep the JSON honest if the launch list changed
        model = [(f"kernel_{j}", 0, 0, 0) for j in range(nl)]
    mean_stage = stage_ms.mean(axis=0)
    stages = []
    for (name, nb, fl, f8), ms in zip(model, mean_stage):
        r = roofline_of(name, nb, fl, float(ms), peaks, f8)
        stages.append({"kernel": name, "ms": round(float(ms), 5),
                       "share": round(float(ms / mean_stage.sum()), 4), **r})
    dom = max(stages, key=lambda d: d["ms"])
    nb = dict((m[0], m) for m in model)[dom["kernel"]]
    roof = {k: dom[k] for k in ("bound", "achieved", "peak", "unit", "frac")}
    roof["kernel"] = dom["kernel"]
    roof["algorithmic"] = nb[1] if dom["bound"] == "hbm" else nb[2]
    roof["peak_source"] = peaks["source"] + (" (burst copy)" if dom["bound"] == "hbm"
                                             else " bf16 burst, fp8 = 2x bf16")
    roof["traffic"] = kernel_traffic(dom["kernel"], f"{shape.name} T={T}")
    wb, wf, w8 = step_work(shape, T, U)
    step_roof = roofline_of("step", wb, wf, ms_step, peaks, w8)
    step_roof.update({"algorithmic_bytes": wb, "algorithmic_flops": wf, "fp8_flops": w8,
                      "note": "whole forward: gate, touched experts, shared expert, fc1/fc2 "
                              "and token rows once, against ms_per_step"})
    return {
        "value": round(value, 2), "ms_per_step": round(ms_step, 5), "path": path,
        "launch": "eager" if graph is None else "cuda_graph_replay", "distinct_experts": U,
        "launches_per_step": nl, "clocks": clk.summary(), "e2e": e2e_rec, "roofline": roof,
        "step_roofline": step_roof, "stages": stages, "stage_timing": STAGE_NOTE,
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="decode", choices=sorted(WORKLOADS))
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--path", default="auto", choices=["auto", "decode", "prefill"],
                    help="force the decode launch or the prefill path (default: the "
                         "library's own choice); a forced path reports no e2e figure")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other workloads' records (measured at N=1 only)")
    ap.add_argument("--eager", action="store_true",
                    help="launch the forward eagerly each step instead of replaying a CUDA graph")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    shape = WORKLOADS[args.workload]
    T = args.tokens or DEFAULT_TOKENS[args.workload]

    if args.impl == "reference":
        run_reference(args, shape, T, rank, world)
        return

    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    flush = L2Flush()
    peaks = measured_peaks()
    inp = make_inputs(shape, T=T)
    rec = measure(inp, T, args, world, flush, peaks)

    subs = []
    if world == 1 and not args.no_workloads:
        cache = {}
        for name, Ts in SUB_WORKLOADS:
            if name == args.workload and Ts == T:
                continue
            if name == args.workload and Ts <= T:
                sub_inp = inp
            else:
                if name not in cache:
                    cache.clear()
                    cache[name] = make_inputs(WORKLOADS[name], T=Ts)
                sub_inp = cache[name]
            # (the workload records take the library's own path choice)
            r = measure(sub_inp, Ts, dataclasses.replace(args, path="auto")
                        if dataclasses.is_dataclass(args) else
                        argparse.Namespace(**{**vars(args), "path": "auto"}), world, flush, peaks)
            subs.append({"workload": config_of(WORKLOADS[name], Ts, r["path"])["workload"],
                         "tokens_per_step": Ts, "metric": METRIC, "unit": UNIT,
                         "dtype": "fp8+bf16" if WORKLOADS[name].expert_fp8 else "bf16",
                         "steps": args.steps, "warmup": args.warmup, **r})
            del sub_inp
        cache.clear()

    if rank == 0:
        line = {
            "metric": METRIC, "value": rec["value"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": rec["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8+bf16" if shape.expert_fp8 else "bf16", "data": "synthetic",
            "config": {**config_of(shape, T, rec["path"]), "global_batch": world * T,
                       "parallelism": f"replicas x{world}",
                       "distinct_experts": rec["distinct_experts"], "launch": rec["launch"]},
            "clocks": rec["clocks"],
            "e2e": rec["e2e"],
            "gpu_launches": rec["launches_per_step"] * args.steps,
            "roofline": rec["roofline"],
            "step_roofline": rec["step_roofline"],
            "stages": rec["stages"],
            "stage_timing": STAGE_NOTE,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(inp, T)
        if subs:
            line["workloads"] = subs
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
