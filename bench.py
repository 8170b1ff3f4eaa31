"""Throughput of the sigmoid-bias top-k MoE feed-forward block on B200.

One step = one forward of the whole block (RMSNorm, router, sigmoid, biased
top-k, dispatch, gate/up + SiLU, down, combine + residual; all 38 blocks for
the stacked workload) over one batch of synthetic tokens already resident in
HBM. Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode]
  python bench.py --impl reference ...   # the fp64 CPU oracle on a bounded sample

Multi-GPU (torchrun, one rank per GPU): every rank runs an independent
replica on its own batch (tokens are independent rows; no collective on the
data path), so per-GPU work is fixed and scaling is weak; the timed region is
bracketed by barriers and the max over ranks is reported.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from sigmoid_bias_top_b200 import accounting as A  # noqa: E402
from sigmoid_bias_top_b200 import workloads as W  # noqa: E402

METRIC = "MoE-layer tokens/s (d2048,E64,top4,I1536) + % of HBM / bf16 TC roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DEFAULT_STEPS = {"decode": 2000, "prefill": 200, "skewed": 100, "stacked": 100, "tiny": 2000,
                 "verify": 1000, "decode_fp8": 2000, "prefill_fp8": 100,
                 "dense_prefill": 100, "dense_decode": 1000, "conv_prefill": 200,
                 "conv_decode": 1000}
# measured after the headline workload in a default one-GPU run
EXTRA = ("prefill,skewed,stacked,verify,decode_fp8,prefill_fp8,"
         "dense_prefill,dense_decode,conv_prefill,conv_decode")
ROTATE = 4  # distinct weight copies cycled through (each step reads >= 1 GB > L2)


# ----------------------------------------------------------------------------- dist
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def reduce_max(v: float, world: int, device=None) -> float:
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(v: float, world: int, device=None) -> float:
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def job_throughput(local_units: float, local_seconds: float, world: int, device=None):
    """Whole-job units/s: units of all ranks over the slowest rank's time."""
    units = reduce_sum(local_units, world, device)
    secs = reduce_max(local_seconds, world, device)
    return units / secs, secs


# ----------------------------------------------------------------------------- peaks
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def traffic_from_profiles(kernel: str, workload: str):
    """dram bytes per launch from the committed ncu summary, if it was taken on
    the kernel source as it is now (source hash recorded in the summary)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    h = re.search(r"source_sha256:\s*([0-9a-f]+)", txt)
    f = re.search(r"source_files:\s*(.+)", txt)
    files = f.group(1).split() if f else None
    if not m or not h or h.group(1) != kernel_source_hash(files):
        return None
    return float(m.group(1))


def _strip_comments(src: str) -> str:
    """C/C++ source without comments and whitespace runs (string literals kept)."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c == '"':
            j = i + 1
            while j < n and src[j] != '"':
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            i = src.find("\n", i)
            i = n if i < 0 else i
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return re.sub(r"\s+", " ", "".join(out)).strip()


def kernel_source_hash(files=None) -> str:
    """Hash of kernel source code (comments and layout ignored): of the given
    csrc files (a kernel's own file and the shared header), else of all of
    them. Recorded with each ncu summary, so that a changed kernel drops its
    traffic figure while changes elsewhere keep it."""
    hs = hashlib.sha256()
    csrc = os.path.join(ROOT, "sigmoid_bias_top_b200", "csrc")
    names = sorted(files) if files else sorted(os.listdir(csrc))
    for f in names:
        if f.endswith((".cu", ".cuh")):
            hs.update(_strip_comments(open(os.path.join(csrc, f), encoding="utf-8").read()).encode())
    return hs.hexdigest()[:16]


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- our arm
KERNEL_PASS_STEPS = 200
KERNEL_MS_NOTE = ("per launch, from a second pass of the same steps (at most "
                  f"{KERNEL_PASS_STEPS}) with CUDA events recorded between the launches, queued "
                  "behind a GPU spin so that the host's launch rate adds no gaps; the events "
                  "break the programmatic-dependent-launch overlap, so each duration includes "
                  "its kernel's start-up")

def make_layers(w, device, n_copies):
    n = w.n_layers if w.n_layers > 1 else n_copies
    return [W.make_layer(w, l, device) for l in range(n)]


def roofline(w, dom, mean_ms, U, peaks, src, clk, timed_s):
    """(bound, work per launch, achieved, peak, unit, peak key) of the
    dominant kernel. Weight-streaming batches (fewer than 64 grouped rows per
    active expert) are bound by HBM; the rest by the tensor cores, against the
    burst bf16 peak unless the clocks saw the power cap or the timed region
    lasted seconds (then the sustained one)."""
    N = w.n_tokens
    n_assign = N * w.top_k
    bpe = 2 if w.dtype == "bf16" else 4
    fp8 = w.dtype == "fp8"
    if n_assign / max(U, 1) < 64:
        if fp8:                  # FP8_BLOCK: both contractions in one launch
            work = A.fp8_experts_bytes(U, n_assign, w.d, w.d_ff)
        elif dom == "experts":   # both contractions in one launch
            work = (A.gate_up_bytes(U, w.d, w.d_ff, bpe) + A.down_bytes(U, w.d, w.d_ff, bpe)
                    + 2 * n_assign * (w.d + w.d_ff) * bpe)
        elif dom == "gate_up":
            work = (A.gate_up_bytes(U, w.d, w.d_ff, bpe) + n_assign * (w.d + w.d_ff) * bpe)
        elif dom == "down":
            work = A.down_bytes(U, w.d, w.d_ff, bpe) + n_assign * (w.d + w.d_ff) * bpe
        else:
            work = A.decode_bytes(U, N, w.d, w.d_ff, w.n_experts, bpe, bpe)
        achieved = work / (mean_ms[dom] / 1e3) / 1e9
        return "hbm", work, achieved, peaks["hbm_gbs"], "GB/s", "hbm_gbs"
    if dom == "experts":
        work = A.gate_up_flops(n_assign, w.d, w.d_ff) + A.down_flops(n_assign, w.d, w.d_ff)
    else:
        work = (A.gate_up_flops(n_assign, w.d, w.d_ff) if dom == "gate_up"
                else A.down_flops(n_assign, w.d, w.d_ff))
    achieved = work / (mean_ms[dom] / 1e3) / 1e12
    sustained = "sw_power_cap" in clk.get("reasons", []) or timed_s >= 1.0
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    peak = peaks.get(key, peaks["bf16_tflops"])
    if fp8:  # e4m3 dense peak = the measured bf16 peak x the nominal 4.5 / 2.25
        peak *= 2.0
        key += " x 2 (e4m3 / bf16 nominal ratio)"
    return "tensor", work, achieved, peak, "TFLOP/s", key


def kernel_pass(step, steps, launches_per_step):
    """The per-kernel pass: the same steps again, with the library recording
    CUDA events between its launches. A GPU spin queued first lets the host
    enqueue the pass's launches and events ahead of the GPU, so each event
    interval times a kernel from the end of the previous one rather than the
    host's launch rate (small batches launch faster on the GPU than the host
    issues them). The events still break the programmatic-dependent-launch
    overlap between kernels."""
    n = min(steps, KERNEL_PASS_STEPS)
    spin_us = min(300_000, 20 * n * launches_per_step)
    torch.cuda._sleep(int(spin_us * 2000))  # ~2 GHz SM clock
    for i in range(n):
        step(i)
    torch.cuda.synchronize()


def measure(w, args, steps, world, rank, local, headline):
    """One workload: W warm-up steps, then `repeats` timed blocks of exactly
    `steps` steps (each bracketed by barrier + synchronize, CUDA events on the
    launching stream); the median block gives the throughput. Then a second,
    separate pass of the same steps with events between the launches gives
    the per-kernel durations. The headline workload also measures the
    end-to-end path through host buffers and the oracle's CPU baseline."""
    from sigmoid_bias_top_b200 import MoeLayer
    dev = torch.device("cuda", local)
    N = w.n_tokens
    layers = make_layers(w, dev, args.rotate)
    mods = [MoeLayer(l, w.top_k, w.eps, w.routed_scale, max_tokens=N) for l in layers]
    n_rot = len(mods) if w.n_layers == 1 else 1
    xs = [W.make_x(w, dev, seed=w.seed + 17 * rank + i) for i in range(max(n_rot, 2))]
    outs = [torch.empty_like(xs[0]) for _ in range(2)]
    stream = torch.cuda.current_stream()

    def step(i, st=None):
        st = stream if st is None else st
        if w.n_layers > 1:  # chained blocks: h = x + MoE(RMSNorm(x))
            h = xs[i % len(xs)]
            for l, m in enumerate(mods):
                dst = outs[l & 1]
                m.forward(h, dst, st)
                h = dst
        else:
            r = i % n_rot
            mods[r].forward(xs[r % len(xs)], outs[i & 1], st)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    for m in mods:
        assert m.status() == 0, m.status()
    graph = None
    if w.n_layers > 1:
        # The stacked decode is timed as one CUDA graph holding all `steps`
        # steps (every launch of the chained layers), replayed once per timed
        # block: its thousands of small launches then cost no host time.
        gs = torch.cuda.Stream(dev)
        gs.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=gs):
            for i in range(steps):
                step(i, gs)
        stream.wait_stream(gs)
        graph.replay()
        torch.cuda.synchronize()
        for m in mods:
            assert m.status() == 0, m.status()

    # routing statistics of the timed batches (distinct active experts per layer)
    active = []
    for r in range(n_rot if w.n_layers == 1 else 1):
        mods[r].forward(xs[r % len(xs)], outs[0], stream)
        off = mods[r].debug_routing(N)["offsets"].cpu().numpy()
        active.append(int((np.diff(off) > 0).sum()))
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.15)
    block_s = []
    for _ in range(args.repeats):
        barrier(world)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        if graph is not None:
            graph.replay()
        else:
            for i in range(steps):
                step(i)
        e1.record(stream)
        torch.cuda.synchronize()
        block_s.append(e0.elapsed_time(e1) / 1e3)
    clk = clocks.stop()
    barrier(world)
    local_s = statistics.median(block_s)
    for m in mods:
        m.profile(True)
    per_step = mods[0].launches_per_forward(N) * (len(mods) if w.n_layers > 1 else 1)
    kernel_pass(step, steps, per_step)
    ktimes = {}
    for m in mods:
        for name, ms in m.kernel_times().items():
            ktimes.setdefault(name, []).append(ms)
        m.profile(False)
        assert m.status() == 0
    value, secs = job_throughput(N * steps, local_s, world, dev)
    per_layer = {k: float(np.mean(v)) for k, v in ktimes.items()}   # per launch
    dom = max(per_layer, key=per_layer.get)
    U = float(np.mean(active))
    peaks, src = load_peaks()
    bound, work, achieved, peak, unit, key = roofline(w, dom, per_layer, U, peaks, src, clk,
                                                      sum(block_s))
    res = {
        "workload": w.name, "value": value, "unit": "tokens/s", "steps": steps,
        "repeats": args.repeats, "ms_per_step": secs / steps * 1e3,
        "ms_per_step_blocks": [b / steps * 1e3 for b in block_s],
        "dtype": "e4m3" if w.dtype == "fp8" else w.dtype,
        "tokens_per_gpu": N, "layers": w.n_layers, "active_experts_per_layer": U,
        "l2": (f"weights rotate over {n_rot} copies; each step streams one copy's active "
               "experts, >= 0.5 GB (> 126 MB L2)" if w.n_layers == 1
               else f"{w.n_layers} distinct layers, {w.n_layers * 1.21:.1f} GB per step (> L2)"),
        "launch": ("one CUDA graph of the timed steps, replayed per block" if graph is not None
                   else "eager launches through the C ABI"),
        "gpu_launches": mods[0].launches_per_forward(N) * steps * args.repeats
                        * (len(mods) if w.n_layers > 1 else 1),
        "roofline": {"bound": bound, "kernel": dom, "achieved": achieved, "peak": peak,
                     "unit": unit, "frac": achieved / peak,
                     "traffic": traffic_from_profiles(dom, args_name(w)),
                     "peak_source": f"{src} ({key})", "work_per_launch": work,
                     "kernel_time": "mean per launch from the separate event-separated pass"},
        "kernel_ms": per_layer,
        "kernel_ms_note": KERNEL_MS_NOTE,
        "clocks": clk,
    }
    if headline:
        # end to end through the C ABI with host buffers (H2D + forward + D2H per step)
        xh = xs[0].cpu().pin_memory()
        oh = torch.empty_like(xh).pin_memory()
        e2e_steps = max(10, min(steps * args.repeats, 500))
        for _ in range(3):
            mods[0].forward_host(xh, oh)
        barrier(world)
        t0 = time.perf_counter()
        for _ in range(e2e_steps):
            if w.n_layers > 1:
                # first block from host, the chain on device, last block back to host
                h = xh.to(dev, non_blocking=True)
                for l, m in enumerate(mods):
                    dst = outs[l & 1]
                    m.forward(h, dst, stream)
                    h = dst
                oh.copy_(h, non_blocking=True)
                torch.cuda.synchronize()
            else:
                mods[0].forward_host(xh, oh)
        e2e_local = time.perf_counter() - t0
        e2e_value, _ = job_throughput(N * e2e_steps, e2e_local, world, dev)
        nbytes = xh.numel() * xh.element_size()
        res["e2e"] = {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": nbytes,
                      "d2h_bytes_per_step": nbytes}
        if rank == 0 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(w, xs[0], layers[0], budget_s=args.cpu_budget)
    for m in mods:
        m.close()
    del mods, layers, xs, outs
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def measure_block(w, args, steps, world, rank, local):
    """A dense or short-convolution block workload: as measure(), with the
    weights and inputs rotated over copies so that every step's weights and
    rows exceed L2 together."""
    from sigmoid_bias_top_b200.blocks import ConvBlock, DenseBlock
    dev = torch.device("cuda", local)
    N = w.n_tokens
    per_copy = (3 * w.d * w.d_ff if w.kind == "dense" else 4 * w.d * w.d) * 2 + 2 * N * w.d * 2
    n_rot = max(2, -(-(3 * 126 * 2 ** 20) // per_copy))  # >= 3x L2 over the rotation
    n_rot = min(n_rot, 8)
    layers = [W.make_block_layer(w, dev, layer=i) for i in range(n_rot)]
    Cls = DenseBlock if w.kind == "dense" else ConvBlock
    mods = [Cls(l, w.eps, max_tokens=N) for l in layers]
    xs = [W.make_block_x(w, dev, seed=w.seed + 17 * rank + i) for i in range(n_rot)]
    outs = [torch.empty_like(xs[0]) for _ in range(2)]
    states = ([W.make_conv_state(w, dev, seed=w.seed + i) for i in range(n_rot)]
              if w.kind == "conv" and w.with_state else None)
    stream = torch.cuda.current_stream()

    def step(i):
        r = i % n_rot
        if w.kind == "dense":
            mods[r].forward(xs[r], outs[i & 1], stream=stream)
        else:
            st = states[r] if states else None
            mods[r].forward(xs[r], outs[i & 1], state_in=st, state_out=st, stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    for m in mods:
        assert m.status() == 0
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.15)
    block_s = []
    for _ in range(args.repeats):
        barrier(world)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(steps):
            step(i)
        e1.record(stream)
        torch.cuda.synchronize()
        block_s.append(e0.elapsed_time(e1) / 1e3)
    clk = clocks.stop()
    barrier(world)
    for m in mods:
        m.profile(True)
    kernel_pass(step, steps, 8)
    ktimes = {}
    for m in mods:
        for name, ms in m.kernel_times().items():
            ktimes.setdefault(name, []).append(ms)
        m.profile(False)
        assert m.status() == 0
    value, secs = job_throughput(N * steps, statistics.median(block_s), world, dev)
    per = {k: float(np.mean(v)) for k, v in ktimes.items()}
    dom = max(per, key=per.get)
    flops, nbytes = A.block_kernel_work(w.kind, dom, N, w.d, w.d_ff)
    peaks, src = load_peaks()
    if w.seq_len > 1:   # prefill: tensor-bound
        sustained = "sw_power_cap" in clk.get("reasons", []) or sum(block_s) >= 1.0
        key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
        bound, work, unit, peak = "tensor", flops, "TFLOP/s", peaks.get(key, peaks["bf16_tflops"])
        achieved = flops / (per[dom] / 1e3) / 1e12
    else:               # decode: weight streaming, HBM-bound
        key = "hbm_gbs"
        bound, work, unit, peak = "hbm", nbytes, "GB/s", peaks["hbm_gbs"]
        achieved = nbytes / (per[dom] / 1e3) / 1e9
    res = {
        "workload": w.name, "value": value, "unit": "tokens/s", "steps": steps,
        "repeats": args.repeats, "ms_per_step": secs / steps * 1e3,
        "ms_per_step_blocks": [b / steps * 1e3 for b in block_s], "dtype": "bf16",
        "tokens_per_gpu": N, "sequences": w.n_seqs, "seq_len": w.seq_len,
        "l2": f"weights and inputs rotate over {n_rot} copies (>= 3x the 126 MB L2)",
        "block_tflops": A.block_flops_per_token(w.kind, w.d, w.d_ff) * N / secs * steps / 1e12,
        "roofline": {"bound": bound, "kernel": dom, "achieved": achieved, "peak": peak,
                     "unit": unit, "frac": achieved / peak,
                     "traffic": traffic_from_profiles(dom, args_name(w)),
                     "peak_source": f"{src} ({key})", "work_per_launch": work,
                     "kernel_time": "mean per launch from the separate event-separated pass"},
        "kernel_ms": per, "kernel_ms_note": KERNEL_MS_NOTE, "clocks": clk,
    }
    for m in mods:
        m.close()
    del mods, layers, xs, outs, states
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def args_name(w):
    """Short workload name (the key of W.WORKLOADS) used by the profile files."""
    for k, v in list(W.WORKLOADS.items()) + list(W.BLOCK_WORKLOADS.items()):
        if v.name == w.name:
            return k
    return w.name


def run_ours(args, w, world, rank, local):
    torch.cuda.set_device(local)
    init_dist(world, "nccl")
    if isinstance(w, W.BlockWorkload):
        # a dense or conv block on its own (profiling runs): its measurement
        # is the line; no host-buffer path or oracle leg
        r = measure_block(w, args, args.steps, world, rank, local)
        r.update({"metric": f"{w.kind} block tokens/s", "n_gpus": world, "warmup": args.warmup,
                  "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                  "data": "synthetic (seeded; random-init weights of the block's shapes)",
                  "config": {"workload": w.name, "parallelism": "single" if world == 1 else
                             f"replicas{world}"}})
        return r
    head = measure(w, args, args.steps, world, rank, local, headline=True)
    line = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "repeats": args.repeats,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": head["dtype"],
        "data": "synthetic (seeded; random-init weights of the layer's shapes)",
        "config": {"workload": w.name, "tokens_per_gpu": w.n_tokens, "layers": w.n_layers,
                   "d": w.d, "experts": w.n_experts, "top_k": w.top_k, "d_ff": w.d_ff,
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": head["l2"], "active_experts_per_layer": head["active_experts_per_layer"],
                   "timing": (f"median of {args.repeats} timed blocks of exactly {args.steps} "
                              "steps, each bracketed by barrier + synchronize")},
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "roofline": head["roofline"],
        "kernel_ms": head["kernel_ms"],
        "kernel_ms_note": head["kernel_ms_note"],
        "ms_per_step_blocks": head["ms_per_step_blocks"],
        "clocks": head["clocks"],
    }
    if "cpu_baseline" in head:
        line["cpu_baseline"] = head["cpu_baseline"]
    # the other configurations, each with its own step count, on one GPU only
    extra = [x for x in args.extra.split(",") if x] if world == 1 else []
    if extra:
        line["workloads"] = {}
        for name in extra:
            if name == args.workload:
                continue
            try:
                if name in W.BLOCK_WORKLOADS:
                    r = measure_block(W.BLOCK_WORKLOADS[name], args, DEFAULT_STEPS[name], world,
                                      rank, local)
                else:
                    r = measure(W.WORKLOADS[name], args, DEFAULT_STEPS[name], world, rank, local,
                                headline=False)
            except Exception as exc:  # one workload's failure must not lose the headline line
                r = {"error": f"{type(exc).__name__}: {exc}"}
                torch.cuda.synchronize()
                torch.cuda.empty_cache()
            line["workloads"][name] = r
    return line


# ----------------------------------------------------------------------------- oracle arm
def cpu_baseline(w, x, layer, budget_s=15.0, tokens_per_call=None):
    """The fp64 oracle as it stands, timed on this host's cores over a bounded
    sample of the workload (whole tokens through the whole layer)."""
    import oracle
    cores = oracle.set_threads(0)
    x_cpu = x.detach().cpu()
    l_cpu = {k: v.detach().cpu() for k, v in layer.items()}
    n = tokens_per_call or min(w.n_tokens, max(1, cores))
    done, t_total, calls = 0, 0.0, 0
    while t_total < budget_s and calls < 1000:
        toks = np.arange(done, done + n) % w.n_tokens
        t0 = time.perf_counter()
        oracle.forward(x_cpu, l_cpu, w.top_k, w.eps, w.routed_scale, tokens=toks)
        t_total += time.perf_counter() - t0
        done += n
        calls += 1
    tps = done / t_total / max(w.n_layers, 1)
    return {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": (f"{done} tokens of {w.name} through one full block (fp64, "
                       f"{calls} calls of {n} tokens, {t_total:.1f} s)"
                       + ("; per-token cost of one block divided by 38 blocks"
                          if w.n_layers > 1 else ""))}


def run_reference(args, w, world, rank):
    if rank != 0:
        return None
    import oracle
    cores = oracle.set_threads(0)
    layer = W.make_layer(w, 0, "cpu")
    x = W.make_x(w, "cpu")
    # each step: a bounded sample (whole tokens through one block), sized so
    # that warm-up + steps stay within about a minute
    probe_t0 = time.perf_counter()
    oracle.forward(x, layer, w.top_k, w.eps, w.routed_scale, tokens=np.arange(min(cores, w.n_tokens)))
    t_tok = (time.perf_counter() - probe_t0) / min(cores, w.n_tokens)
    per_step = max(1, int(60.0 / max(args.steps + args.warmup, 1) / max(t_tok, 1e-9)))
    per_step = min(per_step, w.n_tokens)
    done = 0
    for i in range(args.warmup):
        oracle.forward(x, layer, w.top_k, w.eps, w.routed_scale,
                       tokens=(np.arange(per_step) + i * per_step) % w.n_tokens)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle.forward(x, layer, w.top_k, w.eps, w.routed_scale,
                       tokens=(np.arange(per_step) + i * per_step) % w.n_tokens)
        done += per_step
    secs = time.perf_counter() - t0
    value = done / secs / max(w.n_layers, 1)
    unit = "tokens/s"
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": w.name, "tokens_per_gpu": w.n_tokens, "layers": w.n_layers,
                   "parallelism": "cpu", "sample_tokens_per_step": per_step},
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                         "sample": f"{per_step} tokens per step through one block, fp64"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="decode",
                    choices=sorted(W.WORKLOADS) + sorted(W.BLOCK_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--rotate", type=int, default=ROTATE,
                    help="distinct weight copies cycled through (single-layer workloads)")
    ap.add_argument("--repeats", type=int, default=5,
                    help="timed blocks of --steps steps; the median block is reported")
    ap.add_argument("--extra", default=None,
                    help="comma-separated further workloads measured after the headline "
                         "one on a single GPU (default: all others for decode, none otherwise)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.steps is None:
        args.steps = DEFAULT_STEPS[args.workload]
    if args.extra is None:
        args.extra = EXTRA if args.workload == "decode" else ""
    if args.repeats < 1:
        ap.error("--repeats must be >= 1")
    w = W.WORKLOADS.get(args.workload) or W.BLOCK_WORKLOADS[args.workload]
    world, rank, local = dist_env()
    if args.impl == "reference" and isinstance(w, W.BlockWorkload):
        ap.error("the reference arm times the MoE block's oracle; pick an MoE workload")
    if args.impl == "reference":
        line = run_reference(args, w, world, rank)
    else:
        line = run_ours(args, w, world, rank, local)
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    if world > 1 and torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
