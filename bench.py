#!/usr/bin/env python
"""Benchmark of the MoE-layer forward (top-k routed SwiGLU experts) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill|...]
    python bench.py --impl reference ...     # the fp64 CPU oracle, timed on host cores

One step = one full forward of the layer (router GEMM -> softmax/top-k ->
histogram/offsets -> permutation -> grouped w1/w3 GEMM + SwiGLU -> grouped w2
GEMM + weighted combine) on one batch of seeded synthetic input already
resident in HBM. Rank 0 prints ONE JSON line. With N > 1 (torchrun), every
rank runs an independent replica of the same workload on its own GPU (the
layer has no cross-GPU exchange in this configuration): value = tokens of all
ranks / max-over-ranks device time ("weak" scaling).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time
from dataclasses import replace

import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_mixture_experts_17_b200 import inputs as I  # noqa: E402

METRIC = "MoE-layer tokens/s + active TFLOP/s (prefill), HBM GB/s (decode) vs roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------- distributed plumbing

def dist_setup(use_cuda: bool):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend="nccl" if use_cuda else "gloo",
                                timeout=datetime.timedelta(seconds=180))
    return world, rank, local


def barrier(world):
    if world > 1:
        dist.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                       "-lms", "200", "-i", str(self.gpu)],
                                      stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.p = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.rows = []
        if self.p is None:
            return False
        time.sleep(0.3)
        self.p.terminate()
        try:
            out, _ = self.p.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
            out, _ = self.p.communicate()
        for line in out.splitlines():
            f = [c.strip() for c in line.split(",")]
            if len(f) >= 9:
                self.rows.append(f)
        return False

    def summary(self):
        rows = getattr(self, "rows", [])
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        pw = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [s for s, p in zip(sm, pw) if p is not None and p > 200] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None,
                "reasons": reasons, "samples": len(rows)}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- work accounting

def routed_kept(idx: torch.Tensor, E: int, capacity: int) -> int:
    counts = torch.bincount(idx.flatten().long(), minlength=E)
    if capacity > 0:
        counts = counts.clamp(max=capacity)
    return int(counts.sum().item())


def prefill_flops(w, n_kept):
    ffn = 2.0 * n_kept * 3 * w.d * w.d_ff
    router = 2.0 * w.T * w.d * w.E
    shared = 2.0 * w.T * 3 * w.d * w.d_ff_shared
    return ffn + router + shared, 2.0 * n_kept * w.d * 2 * w.d_ff, 2.0 * n_kept * w.d * w.d_ff


def decode_bytes(w, T, idx):
    U = int(torch.unique(idx.flatten()).numel())
    expert = U * 3 * w.d * w.d_ff * 2
    w13 = U * 2 * w.d * w.d_ff * 2
    other = w.E * w.d * 2 + T * w.d * 2 + T * w.d * 4 + 3 * w.d * w.d_ff_shared * 2
    return U, expert + other, w13, expert


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# the headline kernel, from one ncu capture of the full-size launch; the
# summary, with the command that made it, is under profiles/. `sources_sha`
# is the SHA-256 of what decides that launch when the counters were taken:
# the kernel's sources (TRAFFIC_SOURCES) and the host functions that pick its
# engine and build its tile lists (TRAFFIC_FUNCS). Once any of them changes
# the figure no longer describes the launch, and the line reports null.
TRAFFIC_SOURCES = ["sparse_mixture_experts_17_b200/csrc/gemm_tc.cu",
                   "sparse_mixture_experts_17_b200/csrc/common.cuh",
                   "sparse_mixture_experts_17_b200/csrc/tiles.cuh"]
TRAFFIC_FUNCS = [("sparse_mixture_experts_17_b200/csrc/moe_api.cu", ["use_pair", "set_tiles"])]
TRAFFIC = {
    "prefill": {"bytes": 3373873920 + 931441664, "sources_sha": "e4adf1cb5b4a22bc",
                "kernel": "k_gemm_tc2<EPI_SWIGLU>",
                "profile": "profiles/gemm_w13_traffic_mixtral_t16384.md"},
}


def function_text(src: str, name: str) -> str:
    """The text of top-level function `name` in C++ source `src`: from its
    definition line (starting in column 0) to the first closing brace in
    column 0."""
    m = re.search(r"^[A-Za-z].*\b" + re.escape(name) + r"\(.*$", src, re.M)
    if not m:
        raise KeyError(name)
    end = src.index("\n}\n", m.start())
    return src[m.start():end + 3]


def sources_sha(root: str = ROOT) -> str:
    h = hashlib.sha256()
    for f in TRAFFIC_SOURCES:
        with open(os.path.join(root, f), "rb") as fh:
            h.update(fh.read())
    for f, names in TRAFFIC_FUNCS:
        with open(os.path.join(root, f)) as fh:
            src = fh.read()
        for n in names:
            h.update(function_text(src, n).encode())
    return h.hexdigest()[:16]


def w13_kernel_name(w):
    """The w1/w3 engine the library picks for this workload: the 2-SM pair
    kernel when the experts average >= 1024 routed rows (and 2 d_ff is a
    multiple of 256), else the single-SM kernel."""
    if (w.T * w.k) // w.E >= 1024 and (2 * w.d_ff) % 256 == 0:
        return "k_gemm_tc2<EPI_SWIGLU> (2-SM pair, grouped w1/w3 GEMM + SwiGLU)"
    return "k_gemm_tc<256,EPI_SWIGLU> (grouped w1/w3 GEMM + SwiGLU)"


def headline_traffic(w):
    t = TRAFFIC.get(w.name)
    if not t or t["sources_sha"] != sources_sha() or not w13_kernel_name(w).startswith(t["kernel"]):
        return None
    return t["bytes"]


# ---------------------------------------------------------------- CPU baseline (the oracle)

def cpu_oracle_timing(w, budget_s=15.0, steps=1, warmup=0):
    """The fp64 oracle, as it stands, on a bounded token sample of workload `w`:
    router logits, top-k, histogram/offsets/capacity and the expert FFN with the
    combine, for n sample tokens. Returns (tokens/s, cores, sample text)."""
    from oracle import oracle as O
    threads = O.num_threads()
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = I.make_inputs(w, gen_dev, seed=0)
    oi = I.oracle_arrays(inp)
    del inp

    def run(n):
        sub = dict(oi)
        sub["x"] = oi["x"][:n]
        t0 = time.perf_counter()
        O.forward(sub)
        return time.perf_counter() - t0

    n = max(1, min(w.T, threads))
    t = run(n)
    while t < budget_s / 4 and n < w.T:
        n = min(w.T, int(n * max(2.0, budget_s / max(t, 1e-3) / 2)))
        t = run(n)
    times = [t]
    for _ in range(max(0, steps - 1)):
        times.append(run(n))
    rate = n / statistics.median(times)
    sample = (f"first {n} of {w.T} tokens; router, top-k, offsets (capacity over the sample) and "
              f"expert FFN + combine in fp64 on {threads} OpenMP threads; median of {len(times)}")
    return rate, threads, sample, n


# ---------------------------------------------------------------- our arm

L2_SCRUB_BYTES = 256 << 20   # twice the 126 MB L2


class L2Scrub:
    """A 256 MB buffer written between timed iterations, so that no iteration
    finds the previous one's weights in the 126 MB L2."""

    def __init__(self, dev):
        self.buf = torch.empty(L2_SCRUB_BYTES // 4, dtype=torch.float32, device=dev)

    def __call__(self):
        self.buf.fill_(1.0)


def time_iters_scrubbed(fn, n, stream, scrub, mean=False):
    """Median (or mean) of n iterations, each timed alone by CUDA events on
    `stream`, with the L2 scrubbed before each (outside the events)."""
    evs = []
    for _ in range(n):
        scrub()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    t = [a.elapsed_time(b) for a, b in evs]
    return statistics.mean(t) if mean else statistics.median(t)


def layer_work(w, n_kept, experts_used):
    """Algorithmic FLOPs and bytes of one forward: the FLOPs of the kept rows'
    expert FFNs, the router and the shared expert; the bytes of the weights of
    every expert that has a kept row, the shared expert, W_g, x (bf16) and out
    (fp32). Intermediates (x_perm, H) are not counted: a layer need not write
    them."""
    flops, _, _ = prefill_flops(w, n_kept)
    nbytes = (experts_used * 3 * w.d * w.d_ff * 2 + 3 * w.d * w.d_ff_shared * 2
              + w.E * w.d * 2 + w.T * w.d * 2 + w.T * w.d * 4)
    return flops, nbytes


def fits_l2(w) -> bool:
    """Whether one forward's weights and activations could stay in the 126 MB L2."""
    return (3 * w.E * w.d * w.d_ff * 2 + 3 * w.d * w.d_ff_shared * 2 + w.T * w.d * 6) < 126e6


def config_of(w, world, experts="bf16"):
    """The workload description both arms print."""
    l2 = ("L2 scrubbed (256 MB written) before each timed forward" if fits_l2(w) else
          "inputs larger than L2 (expert weights and activations exceed 126 MB)")
    return {"workload": w.name, "T": w.T, "d_model": w.d, "d_ff": w.d_ff, "E": w.E,
            "k": w.k, "capacity": w.capacity, "d_ff_shared": w.d_ff_shared,
            "zipf_s": w.zipf_s, "seed": 0, "parallelism": f"replicas x{world}",
            "l2": l2, "output": "fp32 [T, d]", "experts": experts}


def time_loop(fn, steps, stream):
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        fn()
    e.record(stream)
    e.synchronize()
    return s.elapsed_time(e) / steps


def run_route_only(a, world, rank, local):
    """Profiling aid: moe_route (the router GEMM with its top-k) alone on the
    workload's x and W_g, K timed calls; no expert weights are allocated.
    Reports GB/s over the bytes the router must read (x, W_g) and write
    (logits, indices, weights)."""
    from sparse_mixture_experts_17_b200 import build as B
    from sparse_mixture_experts_17_b200 import moe as M
    if rank == 0 or not os.path.exists(M.LIB_PATH):
        B.build()
    barrier(world)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peaks, peak_src = load_peaks()
    w = I.WORKLOADS[a.workload]
    if a.tokens:
        w = w.with_T(a.tokens)
    inp = I.make_inputs(w, dev, seed=0, router_only=True)
    s = M.shape_of(w)
    ws = M.alloc_workspace(s, dev)
    logits = torch.empty(w.T, w.E, dtype=torch.float32, device=dev)
    idx = torch.empty(w.T, w.k, dtype=torch.int32, device=dev)
    wts = torch.empty(w.T, w.k, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def step():
        M.moe_route(s, inp["x"], inp["wg"], inp["bias"], logits, idx, wts, status, ws)
    for _ in range(a.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(time_loop(step, a.steps, stream), world, dev)
    nbytes = w.T * w.d * 2 + w.E * w.d * 2 + w.T * w.E * 4 + w.T * w.k * 8
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"metric": "moe_route GB/s (router GEMM + top-k)", "value": round(gbs, 1),
            "unit": "GB/s", "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_of(w, world), "bytes_per_step": nbytes,
            "frac_hbm": round(gbs / peaks["hbm_gbs"], 4), "peak_source": f"{peak_src} hbm_gbs"}


def run_ours(a, world, rank, local):
    from sparse_mixture_experts_17_b200 import build as B
    from sparse_mixture_experts_17_b200 import moe as M
    if rank == 0 or not os.path.exists(M.LIB_PATH):
        B.build()
    barrier(world)
    M.lib()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peaks, peak_src = load_peaks()
    w = I.WORKLOADS[a.workload]
    if a.tokens:
        w = w.with_T(a.tokens)
    if a.experts:
        w = replace(w, E=a.experts, name=f"{w.name}@E{a.experts}",
                    capacity=I.capacity_for(w.T, w.k, a.experts) if w.capacity else 0)
    inp = I.make_inputs(w, dev, seed=0)
    if a.mxfp8 or a.nvfp4:
        # quantize once, then free the bf16 experts: only the block-scaled ones stay resident
        layer = M.MoeLayerMx(inp) if a.mxfp8 else M.MoeLayerNv4(inp)
        for key in ("W1", "W3", "W2", "W1s", "W3s", "W2s"):
            inp.pop(key, None)
        torch.cuda.empty_cache()
        a.no_extra = a.no_e2e = True
    else:
        layer = M.MoeLayer(inp)
    x = inp["x"]
    out = torch.empty(w.T, w.d, dtype=torch.float32, device=dev)
    idx = torch.empty(w.T, w.k, dtype=torch.int32, device=dev)

    for _ in range(a.warmup):
        layer.forward(x, out=out, topk_idx_out=idx)
    torch.cuda.synchronize()
    if int(layer.status.item()) != 0:
        raise RuntimeError(f"device status {int(layer.status.item())} after warm-up")
    n_kept = routed_kept(idx, w.E, w.capacity)

    with ClockSampler(local) as clk:
        # headline: K steps with nothing between the layer's kernels
        launches0 = M.moe_kernel_launches()
        barrier(world)
        torch.cuda.synchronize()
        if fits_l2(w):   # K forwards, each timed alone after an L2 scrub
            scrub = L2Scrub(dev)
            step_ms = time_iters_scrubbed(lambda: layer.forward(x, out=out), a.steps, stream,
                                          scrub, mean=True)
            del scrub
        else:
            step_ms = time_loop(lambda: layer.forward(x, out=out), a.steps, stream)
        torch.cuda.synchronize()
        barrier(world)
        launches = M.moe_kernel_launches() - launches0
        # the same K steps again with CUDA events between the stages (per-kernel times)
        M.moe_profile_enable(True)
        prof_ms = time_loop(lambda: layer.forward(x, out=out), a.steps, stream)
        M.moe_profile_enable(False)
        stages = M.moe_profile_read()
    step_ms_max = max_over_ranks(step_ms, world, dev)
    tokens_all = sum_over_ranks(float(w.T), world, dev)
    value = tokens_all / (step_ms_max / 1e3)

    flops, w13_flops, w2_flops = prefill_flops(w, n_kept)
    # bytes the w1/w3 launch must move: every expert's W13 (all hold rows at
    # this size), the permuted activations read once, H written once
    w13_alg_bytes = int(w.E * 2 * w.d_ff * w.d * 2 + n_kept * w.d * 2 + n_kept * w.d_ff * 2)
    # MXFP8: the fp8 dense peak, twice the measured sustained bf16 figure (the
    # nominal fp8:bf16 ratio; no fp8 peak is measured on this machine)
    ratio = 2.0 if a.mxfp8 else 4.0 if a.nvfp4 else 1.0   # NVFP4: the fp4:bf16 nominal ratio
    # the kernel is timed inside a step of a few ms in a run of well under a
    # second: the burst figure is its peak; the sustained one is reported beside
    peak_t = peaks["bf16_tflops"] * ratio
    stage_ms = {k: round(v[0] / v[1], 4) for k, v in stages.items()}
    decode_path = "dec_w13" in stages
    extra = {}
    if not decode_path:
        w13_ms = stages["w13"][0] / stages["w13"][1]
        w2_ms = stages["w2"][0] / stages["w2"][1]
        ach = w13_flops / (w13_ms / 1e3) / 1e12
        if a.mxfp8 or a.nvfp4:
            fmt = "MXFP8" if a.mxfp8 else "NVFP4"
            nominal = 4500.0 if a.mxfp8 else 9000.0
            roofline = {"bound": "tensor",
                        "kernel": f"k_gemm_mx<EPI_SWIGLU_MX> (block-scaled {fmt} w1/w3 GEMM + SwiGLU)",
                        "achieved": round(ach, 1), "peak": peak_t, "unit": "TFLOP/s",
                        "frac": round(ach / peak_t, 4), "traffic": None,
                        "peak_source": f"{ratio:g} x {peak_src} bf16_tflops (burst; nominal ratio)",
                        "frac_of_sustained": round(ach / (peaks["bf16_tflops_sustained"] * ratio), 4),
                        f"frac_of_nominal_{nominal:.0f}": round(ach / nominal, 4),
                        "algorithmic_flops_per_launch": w13_flops, "avg_launch_ms": round(w13_ms, 4)}
        else:
            roofline = {"bound": "tensor",
                        "kernel": w13_kernel_name(w),
                        "achieved": round(ach, 1), "peak": peak_t, "unit": "TFLOP/s",
                        "frac": round(ach / peak_t, 4), "traffic": headline_traffic(w),
                        "algorithmic_bytes_per_launch": w13_alg_bytes,
                        "peak_source": f"{peak_src} bf16_tflops (burst)",
                        "frac_of_sustained": round(ach / peaks["bf16_tflops_sustained"], 4),
                        "frac_of_nominal_2250": round(ach / 2250.0, 4),
                        "algorithmic_flops_per_launch": w13_flops, "avg_launch_ms": round(w13_ms, 4)}
        extra["w2_tflops"] = round(w2_flops / (w2_ms / 1e3) / 1e12, 1)
        extra["active_tflops"] = round(flops / (step_ms_max / 1e3) / 1e12, 1)
        extra["active_tflops_frac_burst"] = round(flops / (step_ms_max / 1e3) / 1e12 / peak_t, 4)
        extra["n_kept"] = n_kept
    else:
        idx_now = torch.empty(w.T, w.k, dtype=torch.int32, device=dev)
        layer.forward(x, out=out, topk_idx_out=idx_now)
        U, nbytes, w13_bytes, expert_bytes = decode_bytes(w, w.T, idx_now)
        if a.mxfp8 or a.nvfp4:
            # bytes per weight instead of 2: a code byte and 1/32 of a scale
            # byte (MXFP8), or half a code byte and 1/16 of a scale byte (NVFP4)
            mx = ((1.0 + 1.0 / 32.0) if a.mxfp8 else (0.5 + 1.0 / 16.0)) / 2.0
            nbytes = int(nbytes - expert_bytes * (1.0 - mx))
            w13_bytes, expert_bytes = int(w13_bytes * mx), int(expert_bytes * mx)
        k13 = stages["dec_w13"][0] / stages["dec_w13"][1]
        ach = w13_bytes / (k13 / 1e3) / 1e9
        dec_kernel = ("k_dec_w13_mx" if a.mxfp8 else
                      "k_dec_w13_nvtc + k_dec_w13_nvtc_fix (x to NVFP4 in-kernel, tensor-core tiles)"
                      if a.nvfp4 else "k_dec_w13")
        roofline = {"bound": "hbm", "kernel": f"{dec_kernel} (chosen experts' w1/w3 rows + SwiGLU)",
                    "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(ach / peaks["hbm_gbs"], 4), "traffic": None,
                    "peak_source": f"{peak_src} hbm_gbs",
                    "frac_of_nominal_8000": round(ach / 8000.0, 4),
                    "algorithmic_bytes_per_launch": w13_bytes, "avg_launch_ms": round(k13, 4)}
        extra["unique_experts"] = U
        extra["hbm_GB_s_step"] = round(nbytes / (step_ms_max / 1e3) / 1e9, 1)
        extra["hbm_frac_step_measured"] = round(nbytes / (step_ms_max / 1e3) / 1e9 / peaks["hbm_gbs"], 4)

    # ---- end to end through the C ABI with host buffers (H2D + D2H inside)
    e2e = None
    if not a.no_e2e:
        e2e = run_e2e(M, w, layer, x, dev, stream, world, tokens_all, a)

    # ---- decode (T = 1, 2, 4, 8 on the same Mixtral-shape weights)
    decode = None
    graphs = None
    expert_choice = None
    mxfp8 = None
    nvfp4 = None
    backward = None
    configs = None
    if a.workload == "prefill" and not a.no_extra:
        decode = run_decode_set(M, w, layer, x, dev, stream, world, peaks)
        graphs = run_graph_set(M, layer, x, dev)
        expert_choice = run_expert_choice_set(M, w, layer, x, dev, stream, world, peaks,
                                              max(3, a.steps // 2))
        backward = run_backward_set(M, w, inp, layer, dev, stream, world, peaks,
                                    max(3, a.steps // 4))
        mxfp8 = run_lowp_set(M, w, inp, x, dev, stream, world, peaks, max(3, a.steps // 2),
                             "mxfp8")
        nvfp4 = run_lowp_set(M, w, inp, x, dev, stream, world, peaks, max(3, a.steps // 2),
                             "nvfp4")
        # the other workloads, each on its own inputs (the prefill tensors are
        # released first: the fine-grained workload holds 22.6 GB of experts)
        del layer, inp, x, out, idx
        torch.cuda.empty_cache()
        configs = {name: run_config_set(M, name, dev, stream, world, peaks, a.steps)
                   for name in ("tiny", "fine_grained", "capacity")}

    # ---- CPU baseline: the oracle on host cores (rank 0, N = 1 only)
    cpu = None
    if world == 1 and not a.no_cpu_baseline:
        rate, cores, sample, _ = cpu_oracle_timing(w, budget_s=a.cpu_budget)
        cpu = {"value": round(rate, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": sample}

    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(step_ms_max, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "mxfp8 (e4m3 + e8m0/32)" if a.mxfp8 else
                 "nvfp4 (e2m1 + e4m3/16 + f32 per tensor)" if a.nvfp4 else "bf16",
        "data": "synthetic (seeded, N(0,1) x, N(0,0.02) bf16 weights)",
        "config": config_of(w, world, "mxfp8 (moe_forward_mxfp8)" if a.mxfp8 else
                            "nvfp4 (moe_forward_nvfp4)" if a.nvfp4 else "bf16"),
        **extra,
        "stages_ms": stage_ms,
        "profiled_ms_per_step": round(prof_ms, 4),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }
    if graphs is not None:
        res["launch_overhead"] = graphs
    if expert_choice is not None:
        res["expert_choice"] = expert_choice
    if mxfp8 is not None:
        res["mxfp8"] = mxfp8
    if nvfp4 is not None:
        res["nvfp4"] = nvfp4
    if backward is not None:
        res["backward"] = backward
    if configs is not None:
        res["configs"] = configs
    if decode is not None:
        res["decode"] = decode
    if configs is not None or decode is not None:
        res["summary"] = summarize(res)
    return res


def run_e2e(M, w, layer, x, dev, stream, world, tokens_all, a):
    shape_h = M.shape_of(w, M.MOE_FLAG_HOST_IO)
    ws_h = M.alloc_workspace(shape_h, dev)
    x_h = x.cpu().pin_memory()
    out_h = torch.empty(w.T, w.d, dtype=torch.float32).pin_memory()

    def e2e_step():
        M.moe_forward_host(shape_h, x_h, layer.Wg, layer.bias, layer.W13, layer.W2, layer.W13s,
                           layer.W2s, out_h, layer.status, ws_h)
    ws_h = M.alloc_workspace(shape_h, dev)
    x_h = x.cpu().pin_memory()
    out_h = torch.empty(w.T, w.d, dtype=torch.float32).pin_memory()
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = time_loop(e2e_step, max(3, a.steps // 2), stream)
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    return {"value": round(tokens_all / (e2e_ms / 1e3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": x_h.numel() * 2, "d2h_bytes_per_step": out_h.numel() * 4,
            "ms_per_step": round(e2e_ms, 4), "api": "moe_forward_host (pinned host x and out)"}


def run_graph_set(M, layer, x, dev):
    """Launch overhead: the tiny workload and one-token decode, eager vs replay
    of a captured CUDA graph of the same moe_forward call."""
    res = {}
    tiny = I.make_inputs(I.TINY, dev, seed=0)
    cases = {"tiny_T64": (M.MoeLayer(tiny), tiny["x"]), "decode_T1": (layer, x[:1].contiguous())}
    for name, (lay, xin) in cases.items():
        o = torch.empty(xin.shape[0], lay.workload.d, dtype=torch.float32, device=dev)
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(3):
                lay.forward(xin, out=o)
        torch.cuda.current_stream().wait_stream(side)
        eager = time_loop(lambda: lay.forward(xin, out=o), 200, torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            lay.forward(xin, out=o)
        g.replay()
        torch.cuda.synchronize()
        replay = time_loop(g.replay, 200, torch.cuda.current_stream())
        res[name] = {"eager_us": round(eager * 1e3, 2), "graph_replay_us": round(replay * 1e3, 2)}
        del g
    return res


def run_decode_set(M, w, layer, x, dev, stream, world, peaks):
    """Decode (T = 1, 2, 4, 8) on the prefill workload's weights: the median of
    30 forwards, each timed alone with the L2 scrubbed before it, in GB/s over
    the bytes the step must read (the chosen experts' weights, W_g, x, out)."""
    decode = {}
    scrub = L2Scrub(dev)
    for T in I.DECODE_TS:
        xt = x[:T].contiguous()
        it = torch.empty(T, w.k, dtype=torch.int32, device=dev)
        ot = torch.empty(T, w.d, dtype=torch.float32, device=dev)
        for _ in range(5):
            layer.forward(xt, out=ot, topk_idx_out=it)
        torch.cuda.synchronize()
        U, nbytes, w13_bytes, expert_bytes = decode_bytes(w, T, it)
        ms = time_iters_scrubbed(lambda: layer.forward(xt, out=ot), 30, stream, scrub)
        M.moe_profile_enable(True)
        for _ in range(30):
            scrub()
            layer.forward(xt, out=ot)
        torch.cuda.synchronize()
        M.moe_profile_enable(False)
        st = M.moe_profile_read()
        ms = max_over_ranks(ms, world, dev)
        dec = "dec_w13" in st
        s13, s2 = (st["dec_w13"], st["dec_w2"]) if dec else (st["w13"], st["w2"])
        k13 = s13[0] / s13[1]
        k2 = s2[0] / s2[1]
        decode[f"T{T}"] = {
            "path": "decode kernels" if dec else "tensor-core chain",
            "tokens_per_s": round(T * world / (ms / 1e3), 1), "ms_per_step": round(ms, 4),
            "unique_experts": U, "bytes_per_step": nbytes,
            "GB_s": round(nbytes / (ms / 1e3) / 1e9, 1),
            "frac_hbm_measured": round(nbytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
            "frac_hbm_nominal_8000": round(nbytes / (ms / 1e3) / 1e9 / 8000.0, 4),
            "chosen_expert_GB_s_kernels": round(expert_bytes / ((k13 + k2) / 1e3) / 1e9, 1),
            "w13_kernel_GB_s": round(w13_bytes / (k13 / 1e3) / 1e9, 1),
            "timing": "median of 30, L2 scrubbed (256 MB) before each",
            "stages_ms": {k: round(v[0] / v[1], 4) for k, v in st.items()}}
    del scrub
    return decode


def run_config_set(M, name, dev, stream, world, peaks, steps):
    """One of the other measured workloads (tiny, fine_grained, capacity), on its
    own seeded inputs: ms per forward, tokens/s, active TFLOP/s, and the
    fraction of the roof max(FLOPs / burst bf16 peak, bytes / HBM peak) it
    reaches. Workloads whose bytes fit in L2 are timed one forward at a time
    with the L2 scrubbed before each; the others in a loop (their weights
    exceed L2)."""
    w = I.WORKLOADS[name]
    inp = I.make_inputs(w, dev, seed=0)
    layer = M.MoeLayer(inp)
    x = inp["x"]
    out = torch.empty(w.T, w.d, dtype=torch.float32, device=dev)
    idx = torch.empty(w.T, w.k, dtype=torch.int32, device=dev)
    for _ in range(3):
        layer.forward(x, out=out, topk_idx_out=idx)
    torch.cuda.synchronize()
    if int(layer.status.item()) != 0:
        raise RuntimeError(f"device status {int(layer.status.item())} ({name})")
    n_kept = routed_kept(idx, w.E, w.capacity)
    counts = torch.bincount(idx.flatten().long(), minlength=w.E)
    used = int((counts > 0).sum().item())
    flops, nbytes = layer_work(w, n_kept, used)
    small = fits_l2(w)
    if small:
        scrub = L2Scrub(dev)
        ms = time_iters_scrubbed(lambda: layer.forward(x, out=out), max(20, steps), stream, scrub)
        del scrub
    else:
        ms = time_loop(lambda: layer.forward(x, out=out), max(5, steps), stream)
    ms = max_over_ranks(ms, world, dev)
    M.moe_profile_enable(True)
    time_loop(lambda: layer.forward(x, out=out), max(5, steps // 2), stream)
    M.moe_profile_enable(False)
    st = M.moe_profile_read()
    t_compute = flops / (peaks["bf16_tflops"] * 1e12) * 1e3
    t_bytes = nbytes / (peaks["hbm_gbs"] * 1e9) * 1e3
    res = {"T": w.T, "d": w.d, "d_ff": w.d_ff, "E": w.E, "k": w.k, "capacity": w.capacity,
           "d_ff_shared": w.d_ff_shared, "n_kept": n_kept, "experts_used": used,
           "ms_per_step": round(ms, 4), "tokens_per_s": round(w.T * world / (ms / 1e3), 1),
           "active_tflops": round(flops / (ms / 1e3) / 1e12, 1),
           "GB_s": round(nbytes / (ms / 1e3) / 1e9, 1),
           "roof_ms": round(max(t_compute, t_bytes), 4),
           "roof_bound": "tensor" if t_compute >= t_bytes else "hbm",
           "frac_of_roof": round(max(t_compute, t_bytes) / ms, 4),
           "algorithmic_flops": flops, "algorithmic_bytes": nbytes,
           "timing": "median of single forwards, L2 scrubbed before each" if small
                     else "loop; weights exceed L2",
           "stages_ms": {k: round(v[0] / v[1], 4) for k, v in st.items()}}
    if "w13" in st:
        _, f13, f2 = prefill_flops(w, n_kept)
        res["w13_tflops"] = round(f13 / (st["w13"][0] / st["w13"][1] / 1e3) / 1e12, 1)
        res["w2_tflops"] = round(f2 / (st["w2"][0] / st["w2"][1] / 1e3) / 1e12, 1)
    del layer, inp, x, out, idx
    torch.cuda.empty_cache()
    return res


def summarize(res):
    """The headline figures of the five workloads in a few hundred characters,
    printed last in the line."""
    out = {"C3_prefill": {"ms": res["ms_per_step"], "tok_s": res["value"],
                          "w13_frac_burst": res["roofline"]["frac"],
                          "active_tflops": res.get("active_tflops")}}
    for key, tag in (("tiny", "C1_tiny"), ("fine_grained", "C4_fine_grained"),
                     ("capacity", "C5_capacity")):
        c = res.get("configs", {}).get(key)
        if c:
            out[tag] = {"ms": c["ms_per_step"], "tok_s": c["tokens_per_s"],
                        "frac_of_roof": c["frac_of_roof"], "bound": c["roof_bound"]}
    dec = res.get("decode")
    if dec:
        out["C2_decode"] = {k: {"ms": v["ms_per_step"], "frac_hbm": v["frac_hbm_measured"]}
                            for k, v in dec.items()}
    return out


def run_expert_choice_set(M, w, layer, x, dev, stream, world, peaks, steps):
    """Expert-choice routing on the same weights and tokens: each expert takes
    C = T k / E tokens, so the GEMMs process as many rows as top-k routing."""
    C = w.T * w.k // w.E
    s = M.make_shape(w.T, w.d, w.d_ff, w.E, 1, C, w.d_ff_shared, M.MOE_FLAG_EXPERT_CHOICE)
    ws = M.alloc_workspace(s, dev)
    out = torch.empty(w.T, w.d, dtype=torch.float32, device=dev)

    def step():
        M.moe_forward_expert_choice(s, x, layer.Wg, layer.bias, layer.W13, layer.W2, layer.W13s,
                                    layer.W2s, out, layer.status, ws)
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    if int(layer.status.item()) != 0:
        raise RuntimeError(f"device status {int(layer.status.item())} (expert choice)")
    ms = max_over_ranks(time_loop(step, steps, stream), world, dev)
    M.moe_profile_enable(True)
    time_loop(step, steps, stream)
    M.moe_profile_enable(False)
    st = M.moe_profile_read()
    rows = w.E * min(C, w.T)
    w13_flops = 2.0 * rows * w.d * 2 * w.d_ff
    k13 = st["w13"][0] / st["w13"][1]
    return {"capacity_per_expert": C, "rows": rows, "tokens_per_s": round(w.T * world / (ms / 1e3), 1),
            "ms_per_step": round(ms, 4),
            "w13_tflops": round(w13_flops / (k13 / 1e3) / 1e12, 1),
            "w13_frac_measured_sustained": round(w13_flops / (k13 / 1e3) / 1e12
                                                 / peaks["bf16_tflops_sustained"], 4),
            "stages_ms": {k: round(v[0] / v[1], 4) for k, v in st.items()}}


LOWP = {
    # layer class, format, bytes per weight (codes + block-scale share),
    # tensor peak as a multiple of the measured sustained bf16 peak (the nominal ratio)
    "mxfp8": ("MoeLayerMx", "MXFP8 (E4M3, E8M0 scale per 32) weights, x and h; bf16 router",
              1.0 + 1.0 / 32.0, 2.0),
    "nvfp4": ("MoeLayerNv4", "NVFP4 (E2M1, E4M3 scale per 16, fp32 global scale per tensor) "
              "weights, x and h; bf16 router", 0.5 + 1.0 / 16.0, 4.0),
}


def run_lowp_set(M, w, inp, x, dev, stream, world, peaks, steps, fmt):
    """Block-scaled experts (MXFP8 or NVFP4) on the same weights and tokens:
    the prefill step (the w1/w3 GEMM against the format's dense peak, taken as
    the measured sustained bf16 peak times the nominal ratio: 2 for fp8, 4 for
    fp4) and decode at T = 1, 2, 4, 8 (GB/s over the chosen experts' codes and
    scales)."""
    cls, desc, per_weight, ratio = LOWP[fmt]
    lay = getattr(M, cls)(inp)
    out = torch.empty(w.T, w.d, dtype=torch.float32, device=dev)
    idx = torch.empty(w.T, w.k, dtype=torch.int32, device=dev)
    for _ in range(3):
        lay.forward(x, out=out, topk_idx_out=idx)
    torch.cuda.synchronize()
    if int(lay.status.item()) != 0:
        raise RuntimeError(f"device status {int(lay.status.item())} ({fmt})")
    n_kept = routed_kept(idx, w.E, w.capacity)
    ms = max_over_ranks(time_loop(lambda: lay.forward(x, out=out), steps, stream), world, dev)
    M.moe_profile_enable(True)
    time_loop(lambda: lay.forward(x, out=out), steps, stream)
    M.moe_profile_enable(False)
    st = M.moe_profile_read()
    flops, w13_flops, w2_flops = prefill_flops(w, n_kept)
    peak = ratio * peaks["bf16_tflops_sustained"]
    k13 = st["w13"][0] / st["w13"][1]
    k2 = st["w2"][0] / st["w2"][1]
    res = {"format": desc,
           "prefill": {"tokens_per_s": round(w.T * world / (ms / 1e3), 1), "ms_per_step": round(ms, 4),
                       "active_tflops": round(flops / (ms / 1e3) / 1e12, 1),
                       "w13_tflops": round(w13_flops / (k13 / 1e3) / 1e12, 1),
                       "w13_frac_format_peak": round(w13_flops / (k13 / 1e3) / 1e12 / peak, 4),
                       "w2_tflops": round(w2_flops / (k2 / 1e3) / 1e12, 1),
                       "format_peak_tflops": peak,
                       "format_peak_source": f"{ratio:g} x measured bf16_tflops_sustained "
                                             "(nominal ratio)",
                       "stages_ms": {k: round(v[0] / v[1], 4) for k, v in st.items()}}}
    dec = {}
    scrub = L2Scrub(dev)
    for T in I.DECODE_TS:
        xt = x[:T].contiguous()
        it = torch.empty(T, w.k, dtype=torch.int32, device=dev)
        ot = torch.empty(T, w.d, dtype=torch.float32, device=dev)
        for _ in range(5):
            lay.forward(xt, out=ot, topk_idx_out=it)
        torch.cuda.synchronize()
        U = int(torch.unique(it).numel())
        nbytes = int(U * 3 * w.d * w.d_ff * per_weight + w.E * w.d * 2 + T * w.d * 2 + T * w.d * 4)
        # as the bf16 decode: each forward timed alone with the L2 scrubbed
        # before it (the T = 1 codes and scales, ~0.2 GB, are close to L2's size)
        msd = max_over_ranks(time_iters_scrubbed(lambda: lay.forward(xt, out=ot), 30, stream, scrub),
                             world, dev)
        M.moe_profile_enable(True)
        for _ in range(30):
            scrub()
            lay.forward(xt, out=ot)
        torch.cuda.synchronize()
        M.moe_profile_enable(False)
        sd = M.moe_profile_read()
        path = "decode kernels" if "dec_w13" in sd else "tensor-core chain"
        dec[f"T{T}"] = {"path": path, "tokens_per_s": round(T * world / (msd / 1e3), 1),
                        "timing": "median of 30, L2 scrubbed (256 MB) before each",
                        "ms_per_step": round(msd, 4), "unique_experts": U,
                        "bytes_per_step": nbytes, "GB_s": round(nbytes / (msd / 1e3) / 1e9, 1),
                        "frac_hbm_measured": round(nbytes / (msd / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
                        "stages_ms": {k: round(v[0] / v[1], 4) for k, v in sd.items()}}
    res["decode"] = dec
    del lay, scrub
    torch.cuda.empty_cache()
    return res


def run_backward_set(M, w, inp, layer, dev, stream, world, peaks, steps):
    """moe_backward on the same weights and tokens (gradients of sum(out * dout)).
    GEMM FLOPs per step over the n kept rows: the w1/w3 recompute 4 n d d_ff,
    dh 2 n d d_ff, dx 4 n d d_ff, dW2 2 n d d_ff, dW1/dW3 4 n d d_ff."""
    s = M.shape_of(w, M.MOE_FLAG_BACKWARD)
    ws = M.alloc_workspace(s, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    W13T, W2T = M.moe_pack_backward(s, layer.W13, layer.W2)
    g = torch.Generator(dev).manual_seed(1)
    dout = torch.randn(w.T, w.d, generator=g, device=dev)
    x = inp["x"]
    grads = M.moe_backward(s, x, layer.Wg, layer.bias, layer.W13, W13T, W2T, dout, status, ws)

    def step():
        M.moe_backward(s, x, layer.Wg, layer.bias, layer.W13, W13T, W2T, dout, status, ws)
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} (backward)")
    ms = max_over_ranks(time_loop(step, steps, stream), world, dev)
    M.moe_profile_enable(True)
    time_loop(step, steps, stream)
    M.moe_profile_enable(False)
    st = M.moe_profile_read()
    n = w.T * w.k if not w.capacity else None
    if n is None:
        raise RuntimeError("backward measurement expects an uncapped workload")
    flops = 16.0 * n * w.d * w.d_ff
    dw_ms = st["bwd_dw"][0] / st["bwd_dw"][1]
    dh_ms = st["w2"][0] / st["w2"][1]
    del grads, W13T, W2T, ws
    torch.cuda.empty_cache()
    return {"ms_per_step": round(ms, 4), "tokens_per_s": round(w.T * world / (ms / 1e3), 1),
            "gemm_tflops": round(flops / (ms / 1e3) / 1e12, 1),
            "gemm_frac_measured_sustained": round(flops / (ms / 1e3) / 1e12
                                                  / peaks["bf16_tflops_sustained"], 4),
            "dh_tflops": round(2.0 * n * w.d * w.d_ff / (dh_ms / 1e3) / 1e12, 1),
            "weight_grad_stage_tflops": round(6.0 * n * w.d * w.d_ff / (dw_ms / 1e3) / 1e12, 1),
            "stages_ms": {k: round(v[0] / v[1], 4) for k, v in st.items()}}


def run_reference(a, world, rank):
    """The oracle as the reference arm, timed as it stands on the host cores:
    the same metric, unit and config as our arm. Each step is one oracle
    forward of a fixed token sample (router and routing over the sample, the
    expert FFNs and the combine), sized so that the K timed steps take about a
    minute; W warm-up steps run first. value = sample tokens / median step."""
    w = I.WORKLOADS[a.workload]
    from oracle import oracle as O
    O.build()
    threads = O.num_threads()
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = I.make_inputs(w, gen_dev, seed=0)
    oi = I.oracle_arrays(inp)
    del inp

    def step(n):
        sub = dict(oi)
        sub["x"] = oi["x"][:n]
        t0 = time.perf_counter()
        O.forward(sub)
        return time.perf_counter() - t0

    # calibrate the sample: about a.ref_step_s seconds per step
    n = max(1, min(w.T, threads))
    t = step(n)
    while t < a.ref_step_s / 2 and n < w.T:
        n = min(w.T, max(n + 1, int(n * a.ref_step_s / max(t, 1e-3))))
        t = step(n)
    for _ in range(a.warmup):
        step(n)
    times = [step(n) for _ in range(a.steps)]
    med = statistics.median(times)
    rate = n / med
    sample = (f"first {n} of {w.T} tokens per step; router, top-k, offsets (capacity over the "
              f"sample) and expert FFN + combine in fp64 on {threads} OpenMP threads; "
              f"median of {len(times)} steps after {a.warmup} warm-up")
    return {
        "impl": "reference", "metric": METRIC, "value": round(rate, 3), "unit": "tokens/s",
        "n_gpus": world, "steps": len(times), "warmup": a.warmup, "ms_per_step": round(med * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, N(0,1) x, N(0,0.02) bf16 weights)",
        "config": config_of(w, world),
        "sample_tokens_per_step": n,
        "timed_region_s": round(sum(times), 3),
        "cpu_baseline": {"value": round(rate, 3), "unit": "tokens/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(rate, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(I.WORKLOADS), default="prefill")
    ap.add_argument("--no-extra", action="store_true", help="skip the decode measurements")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds per oracle sample")
    ap.add_argument("--ref-step-s", type=float, default=2.5,
                    help="--impl reference: seconds of oracle work per step")
    ap.add_argument("--tokens", type=int, default=0, help="override T (profiling runs)")
    ap.add_argument("--experts", type=int, default=0, help="override E (profiling runs)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end run")
    ap.add_argument("--mxfp8", action="store_true",
                    help="time the layer on MXFP8 experts (moe_forward_mxfp8) instead of bf16; "
                         "no extras, no end-to-end run")
    ap.add_argument("--route-only", action="store_true",
                    help="profiling aid: time moe_route alone (no expert weights allocated)")
    ap.add_argument("--nvfp4", action="store_true",
                    help="time the layer on NVFP4 experts (moe_forward_nvfp4) instead of bf16; "
                         "no extras, no end-to-end run")
    a = ap.parse_args(argv)
    if a.warmup < 3 and a.impl == "ours":
        a.warmup = 3
    if a.impl == "reference":
        world, rank, _ = dist_setup(False)
        if rank != 0:
            return 0
        print(json.dumps(run_reference(a, world, rank)), flush=True)
        return 0
    world, rank, local = dist_setup(True)
    res = run_route_only(a, world, rank, local) if a.route_only else run_ours(a, world, rank, local)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
