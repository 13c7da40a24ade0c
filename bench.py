"""Benchmark of the MoE layer forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one forward pass of the whole layer (router, scan, dispatch, two
grouped GEMMs, combine, losses) over one batch of the workload's synthetic
input, resident in HBM.  L2 is flushed between steps, outside the timed
events: a 256 MiB write, then a 256 MiB read of another buffer.

Default run (no --workload, one GPU): one JSON line per workload on rank 0,
the headline LAST: the Switch layer, the Mixtral-shaped decode layers at
T = 1, 16 and 64 (each timed over at least 100 calls, with the p50 latency
per call), the fine-grained 128-expert layer, and finally the Mixtral-shaped
prefill layer (T 8192, d 4096, 8 experts, top-2, SwiGLU 14336), the largest
single-GPU configuration, whose line also carries a summary of the others.
With --workload NAME, or under torchrun with N > 1, only that workload (the
prefill layer by default) is measured and printed.

--backward times a training step instead (the forward pass, then the
backward pass of <dy, y> + 0.01 aux + 1e-3 z) on one GPU.

N > 1 (torchrun): every rank runs an independent replica of the layer on its
own batch (the layer has no cross-batch exchange), so scaling is weak; the
time is the max over ranks of each rank's device-timed total.
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
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s on 1 B200 and % of roofline (TFLOP/s or HBM GB/s)"
DEFAULT_WORKLOAD = "mixtral_prefill"
# measured before the headline in the default one-GPU run
SECONDARY = ["switch_k1", "mixtral_decode_t1", "mixtral_decode_t16", "mixtral_decode_t64", "fine_grained"]
# (workload, expert weights): the decode layers also with 4-bit weights
SECONDARY_RUNS = [(n, "dense") for n in SECONDARY] + [
    (n, "int4") for n in ("mixtral_decode_t1", "mixtral_decode_t16", "mixtral_decode_t64")]
DECODE_MIN_CALLS = 100  # decode layers report the p50 latency over at least this many calls
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# the nominal B200 figures the layer's targets are quoted against (dense bf16, HBM3e)
NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2200.0}
# Batches of at most this many tokens run the 4-bit layer on the few-row
# products (w4_small_kernel; the first projection's stage also holds
# w4_hidden_kernel), larger ones on the tcgen05 grouped GEMM (w4_gemm_kernel).
W4_SMALL_MAX_T = 64


def w4_kernel_name(T, stage):
    if T > W4_SMALL_MAX_T:
        return "w4_gemm_kernel"
    return "w4_small_kernel + w4_hidden_kernel" if stage == "gemm1" else "w4_small_kernel"


STAGE_KERNEL = {"router": "router_kernel", "scan": "scan_kernel", "dispatch": "dispatch_kernel",
                "gemm1": "grouped_gemm_kernel", "gemm2": "grouped_gemm_kernel", "combine": "combine_kernel"}


# ----------------------------------------------------------------------------- helpers (host only)
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# bytes per weight element of the 4-bit format: half a byte of code plus a
# 2-byte scale per 128 elements
W4_BYTES_PER_WEIGHT = 0.5 + 2.0 / 128


def layer_work(w, kept_counts, weights="dense"):
    """Algorithmic FLOPs and bytes of the layer and of each grouped GEMM launch.

    FLOPs count kept assignments only (plus T rows per shared expert) and the
    router.  Bytes are what the method must move, the expert-sorted
    intermediates (sorted x, hidden activation, fp32 partial rows) excluded:
    the layer reads W_r, the weights of every expert with at least one kept
    row (and of every shared expert) once, x once, and writes y once.  Of
    these, the first projection is charged its weights (W1, and W3 for
    SwiGLU) and x, the second projection its weights (W2) and y.
    """
    elt = 2 if w.dtype == 1 else 4
    welt = W4_BYTES_PER_WEIGHT if weights == "int4" else elt
    n_sh = getattr(w, "n_shared", 0)
    S = int(sum(kept_counts)) + n_sh * w.T
    active = sum(1 for c in kept_counts if c > 0) + n_sh
    nproj1 = 2 if w.act == 1 else 1
    w1_bytes = active * nproj1 * w.d_ff * w.d * welt
    w2_bytes = active * w.d * w.d_ff * welt
    act_bytes = w.T * w.d * elt
    flops_router = 2.0 * w.T * w.E * w.d
    flops1 = 2.0 * S * w.d * w.d_ff * nproj1
    flops2 = 2.0 * S * w.d_ff * w.d
    layer_bytes = w1_bytes + w2_bytes + 2 * act_bytes + w.E * w.d * 4
    return {"S": S, "active_experts": active, "flops_layer": flops_router + flops1 + flops2,
            "bytes_layer": layer_bytes, "gemm1": {"flops": flops1, "bytes": w1_bytes + act_bytes},
            "gemm2": {"flops": flops2, "bytes": w2_bytes + act_bytes}}


def kernel_roofline(flops, nbytes, seconds, peaks):
    """Roofline of one kernel: bound by whichever of its algorithmic FLOPs (at
    the bf16 tensor peak) and bytes (at the HBM bandwidth) takes longer;
    frac against the measured peak, frac_nominal against the nominal one."""
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    if t_tensor >= t_hbm:
        a = flops / seconds / 1e12
        return {"bound": "tensor", "achieved": round(a, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(a / peaks["bf16_tflops"], 4),
                "frac_nominal": round(a / NOMINAL_PEAKS["bf16_tflops"], 4), "algorithmic": flops}
    a = nbytes / seconds / 1e9
    return {"bound": "hbm", "achieved": round(a, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(a / peaks["hbm_gbs"], 4), "frac_nominal": round(a / NOMINAL_PEAKS["hbm_gbs"], 4),
            "algorithmic": nbytes}


def source_sha(*rel):
    h = hashlib.sha256()
    for r in rel:
        with open(os.path.join(ROOT, r), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profiled_traffic(stage, workload, weights="dense"):
    """dram bytes per launch from the committed ncu summary, if the kernel is unchanged since.
    Summaries of the 4-bit kernels carry the suffix _int4."""
    suffix = "_int4" if weights == "int4" else ""
    p = os.path.join(ROOT, "profiles", f"{stage}_{workload}{suffix}.txt")
    if not os.path.exists(p):
        return None
    vals = {}
    with open(p) as f:
        for line in f:
            if ":" in line:
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    src = vals.get("source_files", "").split()
    if not src or "dram_bytes_per_launch" not in vals:
        return None
    if source_sha(*src) != vals.get("source_sha256"):
        return None
    return float(vals["dram_bytes_per_launch"])


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled in the background."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 8:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        win = [p for (t, p) in self.samples if t0 - 0.1 <= t <= t1 + 0.1]
        if not win and self.samples:
            mid = 0.5 * (t0 + t1)
            win = [min(self.samples, key=lambda s: abs(s[0] - mid))[1]]
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for p in win for i in range(4) if p[4 + i].lower().startswith("active")})

        def num(s):
            try:
                return float(s)
            except ValueError:
                return None
        sm = [num(p[1]) for p in win if num(p[1]) is not None]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": num(win[0][2]),
                "power_w_max": max((num(p[3]) or 0.0) for p in win), "reasons": reasons, "samples": len(win)}


def combine_ranks(seconds_local, tokens_local, dist_mod=None):
    """(max over ranks of the timed seconds, sum over ranks of the tokens)."""
    if dist_mod is None or not dist_mod.is_initialized():
        return seconds_local, tokens_local
    import torch
    dev = "cuda" if dist_mod.get_backend() == "nccl" else "cpu"
    t = torch.tensor([seconds_local], dtype=torch.float64, device=dev)
    n = torch.tensor([float(tokens_local)], dtype=torch.float64, device=dev)
    dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    dist_mod.all_reduce(n, op=dist_mod.ReduceOp.SUM)
    return float(t.item()), float(n.item())


def gpu_hold(torch, ms):
    """Keep the GPU busy for about `ms` so the host can enqueue the timed steps
    ahead of it; the step events then measure GPU time only (launch latency of
    the host never shows up as idle GPU time inside a step)."""
    torch.cuda._sleep(int(ms * 2.0e6))  # cycles at ~2 GHz


def rank_seed(base_seed, rank):
    """Each replica draws its own batch of tokens; weights are shared."""
    return base_seed + 7919 * rank


def config_of(w, n_gpus):
    return {"workload": w.name, "T": w.T, "d": w.d, "E": w.E, "k": w.k, "d_ff": w.d_ff, "n_shared": w.n_shared,
            "act": "swiglu" if w.act == 1 else "relu", "gate": "renorm" if w.gate == 1 else "switch",
            "capacity_factor": w.capacity_factor, "tokens_per_gpu": w.T,
            "parallelism": "replicas" if n_gpus > 1 else "single",
            "l2": "flushed between steps outside the timed events: a 256 MiB write, then a 256 MiB read of "
                  "another buffer (the write's dirty lines go back to HBM before the step starts)"}


# ----------------------------------------------------------------------------- CPU (oracle) leg
# Rows of y per host thread in one CPU-baseline sample (the routing always covers
# every token): a few seconds of plain C++ loops per workload.
CPU_ROWS_PER_THREAD = {"switch_k1": 256, "mixtral_prefill": 4, "fine_grained": 64, "fine_grained_shared": 48,
                       "tiny_fp32": 64}


class CpuOracle:
    """The C++ loop oracle on one workload's inputs, copied to host memory once."""

    def __init__(self, w, inp):
        from oracle import cpp
        self.w = w
        self.O = cpp.load()
        self.host = {k: (None if v is None else v.detach().cpu()) for k, v in inp.items()}
        self.hw_threads = self.O.hardware_threads() or (os.cpu_count() or 1)

    def run(self, rows, threads):
        """Seconds of one oracle forward: routing, capacity and losses over all T
        tokens, y for the listed rows."""
        w, h = self.w, self.host
        shared = None
        if w.n_shared:
            ids = slice(w.E, w.E + w.n_shared)
            shared = (h["W1"][ids], None if h["W3"] is None else h["W3"][ids], h["W2"][ids])
        t0 = time.perf_counter()
        self.O.moe_forward(h["x"], h["W_r"], h["b_r"], h["W1"], h["W3"], h["W2"], k=w.k, gate_mode=w.gate,
                           act=w.act, capacity_factor=w.capacity_factor, rows=rows, shared=shared, threads=threads)
        return time.perf_counter() - t0

    def sample_rows(self, per_thread, threads):
        n = min(self.w.T, max(1, per_thread * threads))
        return list(range(n)), n


def layer_rate(T, t_route, t_sample, n):
    """Tokens/s of the whole layer on the host, from the seconds of routing all T
    tokens (t_route) and of routing plus y for n of them (t_sample): y of the
    other T - n tokens costs the same per row."""
    per_row = max(t_sample - t_route, 0.0) / max(n, 1)
    return T / (t_route + per_row * T)


def cpu_baseline(w, inp):
    """The C++ oracle timed on the host cores, as tokens/s of the whole layer:
    all hardware threads over tokens (the reported value), and one thread."""
    co = CpuOracle(w, inp)
    per = CPU_ROWS_PER_THREAD.get(w.name, w.T)
    nt = co.hw_threads
    out = {}
    for threads, rows_per in ((nt, per), (1, max(1, per // 8))):
        rows, n = co.sample_rows(rows_per, threads)
        t_route = co.run([], threads)
        t_sample = co.run(rows, threads)
        out[threads] = (layer_rate(w.T, t_route, t_sample, n), n, t_route, t_sample)
    v, n, tr, ts = out[nt]
    v1, n1, tr1, ts1 = out[1]
    return {"value": round(v, 3), "unit": "tokens/s", "cores": nt, "kind": "oracle",
            "single_thread_value": round(v1, 3),
            "sample": f"C++ loop oracle (oracle/moe_oracle.cpp, float64), {nt} threads over tokens: routing, "
                      f"capacity and losses of all {w.T} tokens ({tr:.2f} s), plus y of the first {n} tokens "
                      f"({ts - tr:.2f} s more), the y rows extrapolated to all {w.T}; single_thread_value: the same "
                      f"on 1 thread with y of {n1} tokens ({tr1:.2f} s + {ts1 - tr1:.2f} s)"}


# ----------------------------------------------------------------------------- GPU leg
def measure_workload(args, w, dev, world, rank, local, K, warmup, cpu=True, weights="dense"):
    """Time K forward passes of workload w (inputs resident in HBM), the
    per-stage breakdown in an untimed pass, and the end-to-end path with
    pinned host buffers.  weights "int4": the experts' weights quantized to
    the 4-bit format once, before any timing (moe_forward_w4).  Returns the
    JSON line (rank 0) or None."""
    import torch
    import torch.distributed as dist
    from sparse_mixture_experts_gating_b200 import MoELayer, launch_count, quantize_int4, status
    from sparse_mixture_experts_gating_b200.workloads import make_inputs, torch_dtype

    decode = w.name.startswith("mixtral_decode")
    if decode:
        K = max(K, DECODE_MIN_CALLS)
    inp = make_inputs(w, device=dev)
    if rank > 0:
        inp["x"] = make_inputs(w.with_(seed=rank_seed(w.seed, rank)), device=dev, weights=False)["x"]
    layer = MoELayer(w.E, w.k, w.d, w.d_ff, act=w.act, gate_mode=w.gate, capacity_factor=w.capacity_factor,
                     dtype=torch_dtype(w.dtype), hidden=args.hidden, n_shared=w.n_shared)
    w4 = weights == "int4"
    if w4:
        qw = {k: (None if inp[k] is None else quantize_int4(inp[k])) for k in ("W1", "W3", "W2")}
        status()
        inp["W1"] = inp["W3"] = inp["W2"] = None  # only the 4-bit copies stay resident
        torch.cuda.empty_cache()
        ws = torch.empty(max(layer.workspace_bytes_w4(w.T), 256), dtype=torch.uint8, device=dev)
    else:
        ws = layer.workspace(w.T, dev)
    y = torch.empty((w.T, w.d), dtype=inp["x"].dtype, device=dev)
    stats = (torch.empty(w.E, dtype=torch.int32, device=dev), torch.empty(1, dtype=torch.int32, device=dev),
             torch.empty(1, dtype=torch.float32, device=dev), torch.empty(1, dtype=torch.float32, device=dev))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_rd = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)

    def flush_l2():
        # a write larger than L2, then a read of another buffer larger than L2:
        # the write's dirty lines are written back here, outside the timed
        # events, and the step starts with L2 holding none of its inputs
        flush.zero_()
        flush_rd.sum()
    stream = torch.cuda.current_stream()
    args_fw = (inp["x"], inp["W_r"], inp["b_r"], inp["W1"], inp["W3"], inp["W2"])

    def step(events=None, x=None):
        a = args_fw if x is None else (x,) + args_fw[1:]
        if w4:
            layer.forward_w4(a[0], a[1], a[2], qw["W1"], qw["W3"], qw["W2"], out=y, stats=stats, workspace=ws,
                             events=events)
        else:
            layer(*a, out=y, stats=stats, workspace=ws, events=events)

    for _ in range(warmup):
        flush_l2()
        step()
    status()

    stage_names = ["router", "scan", "dispatch", "gemm1", "gemm2", "combine"]
    active = [n for n in stage_names
              if not (n == "combine" and w.dtype == 1 and w.k == 1 and w.n_shared == 0 and not w4)]

    # Untimed profiling pass: every stage bracketed by events -> per-kernel breakdown.
    Kp = min(K, 20)
    ev_stage = [[torch.cuda.Event(enable_timing=True) for _ in range(12)] for _ in range(Kp)]
    torch.cuda.synchronize()
    gpu_hold(torch, 2.0 + 0.3 * Kp)
    for i in range(Kp):
        flush_l2()
        step(events=ev_stage[i])
    torch.cuda.synchronize()
    stage_ms = {}
    for s_i, name in enumerate(stage_names):
        if name in active:
            stage_ms[name] = statistics.mean(ev[2 * s_i].elapsed_time(ev[2 * s_i + 1]) for ev in ev_stage)
    dom = max(("gemm1", "gemm2"), key=lambda n: stage_ms[n])
    dom_i = stage_names.index(dom)

    # Timed region: step events, plus the dominant kernel's own pair (live roofline).
    ev_step = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    ev_dom = [[None] * 12 for _ in range(K)]
    for i in range(K):
        ev_dom[i][2 * dom_i] = torch.cuda.Event(enable_timing=True)
        ev_dom[i][2 * dom_i + 1] = torch.cuda.Event(enable_timing=True)
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    sampler = ClockSampler(vis.split(",")[local].strip() if vis else str(local))
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    n_launch0 = launch_count()
    wall0 = time.time()
    gpu_hold(torch, 2.0 + 0.2 * K)
    for i in range(K):
        flush_l2()
        ev_step[i][0].record(stream)
        step(events=ev_dom[i])
        ev_step[i][1].record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    if world > 1:
        dist.barrier()
    n_launch = launch_count() - n_launch0
    time.sleep(0.15)
    sampler.stop()
    status()

    step_ms = [a.elapsed_time(b) for a, b in ev_step]
    total_s = sum(step_ms) / 1e3
    dom_ms = statistics.mean(ev[2 * dom_i].elapsed_time(ev[2 * dom_i + 1]) for ev in ev_dom)

    # end to end through the public API: pinned host x in, y and statistics out, every step
    x_host = inp["x"].cpu().pin_memory()
    y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    st_host = [torch.empty(s.shape, dtype=s.dtype).pin_memory() for s in stats]
    x_dev = torch.empty_like(inp["x"])
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    torch.cuda.synchronize()
    gpu_hold(torch, 2.0 + 0.2 * (K + warmup))
    for i in range(warmup + K):
        flush_l2()
        if i >= warmup:
            e2e_ev[i - warmup][0].record(stream)
        x_dev.copy_(x_host, non_blocking=True)
        step(x=x_dev)
        y_host.copy_(y, non_blocking=True)
        for h, s_ in zip(st_host, stats):
            h.copy_(s_, non_blocking=True)
        if i >= warmup:
            e2e_ev[i - warmup][1].record(stream)
    torch.cuda.synchronize()
    status()
    e2e_ms = [a.elapsed_time(b) for a, b in e2e_ev]
    e2e_s = sum(e2e_ms) / 1e3

    t_max, tokens = combine_ranks(total_s, w.T * K, dist if world > 1 else None)
    e2e_max, _ = combine_ranks(e2e_s, w.T * K, dist if world > 1 else None)

    counts = stats[0].cpu().tolist()
    cap = layer.capacity(w.T)
    kept = [c if cap is None else min(c, cap) for c in counts]
    work = layer_work(w, kept, "int4" if w4 else "dense")
    peaks, peak_src = load_peaks()
    roof = kernel_roofline(work[dom]["flops"], work[dom]["bytes"], dom_ms / 1e3, peaks)
    roof["kernel"] = f"{w4_kernel_name(w.T, dom) if w4 else STAGE_KERNEL[dom]} ({dom})"
    roof["peak_source"] = f"{peak_src} ({'bf16_tflops' if roof['bound'] == 'tensor' else 'hbm_gbs'}, burst)"
    roof["nominal_peak"] = NOMINAL_PEAKS["bf16_tflops" if roof["bound"] == "tensor" else "hbm_gbs"]
    tr = profiled_traffic(dom, w.name, "int4" if w4 else "dense")
    roof["traffic"] = tr
    gemm_bytes = work[dom]["bytes"]
    roof["traffic_ratio"] = None if tr is None else round(tr / gemm_bytes, 3)
    roof["kernel_ms"] = round(dom_ms, 5)
    ms_step = total_s / K * 1e3
    floor_s = max(work["flops_layer"] / (peaks["bf16_tflops"] * 1e12), work["bytes_layer"] / (peaks["hbm_gbs"] * 1e9))
    floor_nom = max(work["flops_layer"] / (NOMINAL_PEAKS["bf16_tflops"] * 1e12),
                    work["bytes_layer"] / (NOMINAL_PEAKS["hbm_gbs"] * 1e9))
    clocks = sampler.summary(wall0, wall1)

    line = None
    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(tokens / t_max, 1),
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": K,
            "warmup": warmup,
            "ms_per_step": round(ms_step, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16" if w.dtype == 1 else "f32",
            "data": "synthetic (seeded; shapes and distributions of the workload, random-init weights)",
            "config": dict(config_of(w, world), hidden=args.hidden,
                           **({"weights": "int4 (codes + bf16 scale per 128; quantized before timing)"}
                              if w4 else {})),
            "roofline": roof,
            "layer_roofline": {"floor_ms": round(floor_s * 1e3, 5), "frac": round(floor_s / (ms_step / 1e3), 4),
                               "floor_ms_nominal": round(floor_nom * 1e3, 5),
                               "frac_nominal": round(floor_nom / (ms_step / 1e3), 4),
                               "flops": work["flops_layer"], "bytes": work["bytes_layer"],
                               "kept_assignments": work["S"], "active_experts": work["active_experts"]},
            "kernels_ms": {k: round(v, 5) for k, v in stage_ms.items()},
            "e2e": {"value": round(tokens / e2e_max, 1), "unit": "tokens/s",
                    "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
                    "d2h_bytes_per_step": y_host.numel() * y_host.element_size()
                    + sum(h.numel() * h.element_size() for h in st_host)},
            "gpu_launches": int(n_launch),
            "clocks": clocks,
        }
        if decode:
            line["latency_ms"] = {"p50": round(statistics.median(step_ms), 5), "min": round(min(step_ms), 5),
                                  "max": round(max(step_ms), 5), "calls": K,
                                  "e2e_p50": round(statistics.median(e2e_ms), 5)}
        if args.hidden == "bf16":
            line["note"] = "hidden activation in one bf16 plane: outside the parity bar"
        if world == 1 and cpu and not args.no_cpu_baseline and not w4:
            line["cpu_baseline"] = cpu_baseline(w, inp)
    del inp, ws, y, flush, flush_rd, x_host, y_host, x_dev
    if w4:
        del qw
    layer = None
    torch.cuda.empty_cache()
    return line


def summary_of(line):
    """The few numbers of a workload's line that the headline line repeats."""
    out = {"tokens_per_s": line["value"], "ms_per_step": line["ms_per_step"],
           "dominant": line["roofline"]["kernel"], "dominant_bound": line["roofline"]["bound"],
           "dominant_frac": line["roofline"]["frac"], "dominant_frac_nominal": line["roofline"]["frac_nominal"],
           "layer_frac": line["layer_roofline"]["frac"], "layer_frac_nominal": line["layer_roofline"]["frac_nominal"],
           "e2e_tokens_per_s": line["e2e"]["value"], "sm_mhz": line["clocks"].get("sm_mhz"),
           "clock_reasons": line["clocks"].get("reasons")}
    if "weights" in line["config"]:
        out["weights"] = "int4"
    if "latency_ms" in line:
        out["p50_ms"] = line["latency_ms"]["p50"]
        out["calls"] = line["latency_ms"]["calls"]
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None,
                    help="measure only this workload (default: every workload, the Mixtral prefill layer last)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--hidden", choices=["auto", "f16", "bf16x2", "bf16"], default="auto",
                    help="how the expert hidden activation is held (bf16 layers; auto: the library's choice)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's token count (small cases for profiler captures)")
    ap.add_argument("--backward", action="store_true",
                    help="time a training step instead: the forward pass, then the backward pass")
    ap.add_argument("--weights", choices=["dense", "int4"], default="dense",
                    help="expert weights: the layer dtype, or the 4-bit format (moe_forward_w4)")
    args = ap.parse_args()

    import torch
    import torch.distributed as dist
    from sparse_mixture_experts_gating_b200.workloads import WORKLOADS, make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    name = args.workload or DEFAULT_WORKLOAD
    w = WORKLOADS[name]
    if args.tokens is not None:
        w = w.with_(T=args.tokens, x_rows_of=None)
    warmup = max(3, args.warmup)

    if args.impl == "reference":
        if rank != 0:
            return 0
        return reference_arm(args, w, warmup)

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)

    if args.backward:
        return backward_bench(args, w, make_inputs(w, device=dev), warmup, world, rank, local, dev)
    others = []
    if args.workload is None and args.tokens is None and world == 1:
        for other, wts in SECONDARY_RUNS:
            line = measure_workload(args, WORKLOADS[other], dev, world, rank, local, args.steps, warmup,
                                    weights=wts)
            print(json.dumps(line), flush=True)
            others.append(line)
    line = measure_workload(args, w, dev, world, rank, local, args.steps, warmup, weights=args.weights)
    if rank == 0:
        if others:
            line["workloads"] = {o["config"]["workload"] + ("_int4" if "weights" in o["config"] else ""):
                                 summary_of(o) for o in others}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def backward_work(w, S, T, active):
    """Algorithmic work of the backward pass for S kept rows (shared rows
    included) and `active` experts with rows.  FLOPs: per row and d x d_ff
    contraction 2 d d_ff, 5 of them for ReLU (w1 x again, W2^T dy, dXp, dW2,
    dW1) and 8 for SwiGLU (w3 x, a second dXp term, dW3 more), plus the
    router's 3 T E d (logits again, W_r^T dh, dW_r).  Bytes: the active
    experts' weights read once, the fp32 weight gradients of every expert
    written once (zeros where no row came), x and dy read, dx and dW_r written."""
    swiglu = w.act == 1
    n_sh = getattr(w, "n_shared", 0)
    flops = 2.0 * S * w.d * w.d_ff * (8 if swiglu else 5) + 3 * 2.0 * T * w.E * w.d
    elt = 2 if w.dtype == 1 else 4
    nproj = 3 if swiglu else 2
    per = nproj * w.d * w.d_ff
    nbytes = (active * per * elt + (w.E + n_sh) * per * 4 + 2 * T * w.d * elt + T * w.d * 4 + w.E * w.d * 4)
    return flops, nbytes


def backward_bench(args, w, inp, warmup, world, rank, local, dev):
    """Training step = forward + backward (gradients of <dy, y> + 0.01 aux +
    1e-3 z), inputs resident, L2 flushed before each step outside the events."""
    import torch
    from sparse_mixture_experts_gating_b200 import MoELayer, launch_count, status
    from sparse_mixture_experts_gating_b200.workloads import torch_dtype
    if world > 1 or rank > 0:
        raise SystemExit("--backward runs on one GPU")
    layer = MoELayer(w.E, w.k, w.d, w.d_ff, act=w.act, gate_mode=w.gate, capacity_factor=w.capacity_factor,
                     dtype=torch_dtype(w.dtype), hidden=args.hidden, n_shared=w.n_shared)
    ws = layer.workspace(w.T, dev)
    gen = torch.Generator().manual_seed(w.seed + 17)
    dy = torch.randn(w.T, w.d, generator=gen).to(inp["x"].dtype).to(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_rd = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)

    def flush_l2():  # as in the forward bench: a write, then a read of another buffer, both larger than L2
        flush.zero_()
        flush_rd.sum()
    fw = (inp["x"], inp["W_r"], inp["b_r"], inp["W1"], inp["W3"], inp["W2"])
    grads = None
    stream = torch.cuda.current_stream()

    def step(ev=None):
        nonlocal grads
        y, counts, *_ = layer(*fw, workspace=ws)
        if ev is not None:
            ev.record(stream)
        grads = layer.backward(*fw, dy, aux_coef=0.01, z_coef=1e-3, workspace=ws, grads=grads)
        return counts

    for _ in range(warmup):
        flush_l2()
        step()
    status()
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    sampler = ClockSampler(vis.split(",")[local].strip() if vis else str(local))
    sampler.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    n0 = launch_count()
    wall0 = time.time()
    gpu_hold(torch, 2.0 + 2.0 * K)
    for i in range(K):
        flush_l2()
        evs[i][0].record(stream)
        counts = step(evs[i][1])
        evs[i][2].record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    n_launch = launch_count() - n0
    time.sleep(0.15)
    sampler.stop()
    status()
    step_s = sum(e[0].elapsed_time(e[2]) for e in evs) / 1e3
    bw_s = sum(e[1].elapsed_time(e[2]) for e in evs) / 1e3
    cap = layer.capacity(w.T)
    kept = sum(c if cap is None else min(c, cap) for c in counts.cpu().tolist())
    S = kept + w.n_shared * w.T
    active = sum(1 for c in counts.cpu().tolist() if c > 0) + w.n_shared
    fl, nb = backward_work(w, S, w.T, active)
    clocks = sampler.summary(wall0, wall1)
    peaks, peak_src = load_peaks()
    t_bw = bw_s / K
    if w.dtype == 1:  # bf16: every product on the tensor cores
        roof = kernel_roofline(fl, nb, t_bw, peaks)
        roof["peak_source"] = f"{peak_src} ({'bf16_tflops' if roof['bound'] == 'tensor' else 'hbm_gbs'}, burst)"
    else:  # fp32: every product on the CUDA cores
        peak = 148 * 128 * 2 * (clocks["sm_max_mhz"] or 1965.0) * 1e6 / 1e12  # fp32 FMA lanes x 2 x max clock
        ach = fl / t_bw / 1e12
        roof = {"bound": "alu", "achieved": round(ach, 2), "peak": round(peak, 1), "unit": "TFLOP/s",
                "frac": round(ach / peak, 4), "peak_source": "148 SMs x 128 fp32 lanes x 2 FLOP x clocks.max.sm"}
    roof["kernel"] = "backward pass (all its launches)"
    roof["traffic"] = None
    line = {
        "metric": "MoE-layer training step (forward + backward) tokens/s on 1 B200",
        "value": round(w.T * K / step_s, 1),
        "unit": "tokens/s",
        "n_gpus": 1,
        "steps": K,
        "warmup": warmup,
        "ms_per_step": round(step_s / K * 1e3, 5),
        "backward_ms": round(bw_s / K * 1e3, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == 1 else "f32",  # operands of the products (bf16 as hi + lo pairs where fp32-derived)
        "data": "synthetic (seeded; shapes and distributions of the workload, random-init weights)",
        "config": dict(config_of(w, 1), hidden=args.hidden, loss="<dy, y> + 0.01 aux + 1e-3 z"),
        "roofline": roof,
        "backward_work": {"flops": fl, "bytes": nb, "kept_rows": S, "active_experts": active},
        "gpu_launches": int(n_launch),
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def reference_arm(args, w, warmup):
    """The C++ loop oracle timed on the host cores (rank 0 only): the reference
    arm of this benchmark.  Each step routes all T tokens and computes y for a
    bounded sample of them (one row per hardware thread at most)."""
    import torch
    from sparse_mixture_experts_gating_b200.workloads import make_inputs

    inp = make_inputs(w, device="cuda" if torch.cuda.is_available() else "cpu")
    co = CpuOracle(w, inp)
    del inp
    nt = co.hw_threads
    per = 1 if w.name in ("mixtral_prefill",) else max(1, CPU_ROWS_PER_THREAD.get(w.name, w.T) // 8)
    rows, n = co.sample_rows(per, nt)
    t_route = min(co.run([], nt) for _ in range(warmup))
    secs = [co.run(rows, nt) for _ in range(args.steps)]
    total = sum(secs)
    value = layer_rate(w.T, t_route, total / args.steps, n)
    line = {
        "metric": METRIC, "impl": "reference", "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps, "warmup": warmup,
        "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": dict(config_of(w, int(os.environ.get("WORLD_SIZE", "1"))), hidden=args.hidden),
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": nt, "kind": "oracle",
                         "sample": f"each step: C++ loop oracle (float64), {nt} threads over tokens, routing all "
                                   f"{w.T} tokens and computing y for the first {n}; value: tokens/s of the whole "
                                   f"layer, y rows extrapolated to all {w.T} (routing alone: {t_route:.3f} s)"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
