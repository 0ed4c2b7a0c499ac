#!/usr/bin/env python
"""Benchmark of the extreme-low-bit linear layer forward on B200.

Headline workload (one "step"): the M=1 decode step over a LLaMA-7B-shaped
stack of ternary BitLinear layers -- 32 blocks x (q, k, v, o: 4096->4096;
gate, up: 4096->11008; down: 11008->4096) = 224 layers with a decode step's
dependencies, run as ONE decode-chain launch (bl_chain_run: each layer
quantises its fp16 input token to int8 and contracts it with 2-bit packed
weights; 1,619,001,344 weight bytes per step, far above the 126 MB L2, so no
flush is needed between steps).  The step is captured once as a CUDA graph and
replayed.  The e2e figure runs the same step through bl_chain_run_host (host
buffers, copies inside the timed region).

Metric: effective packed-weight GB/s at M=1 (and, in the ``prefill`` object,
int8 TOPS at M=512 on LLaMA-70B-shaped layers), each with its roofline
fraction.  Extra objects: the same stack without dependencies, with RMSNorm
and SwiGLU fused, in OneBit form, as separate per-layer calls; the SVID of a
4096x4096 layer; single-layer and batch sweeps (BitLinear, OneBit, BiLLM).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
       python bench.py --case NAME   (one small workload, for ncu profiles)
Multi-GPU (torchrun): independent replicas, no collective on the data path.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

LLAMA7B_BLOCK = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
                 ("gate", 4096, 11008), ("up", 4096, 11008), ("down", 11008, 4096)]  # (name, K, N)
LLAMA7B_LAYERS = 32
LLAMA13B_SWEEP = [("up", 5120, 13824), ("down", 13824, 5120)]   # (name, K, N)
SWEEP_M = [1, 4, 16, 64, 256, 1024]
LLAMA70B_PREFILL = [("qkvo-like", 8192, 8192), ("gate/up", 8192, 28672), ("down", 28672, 8192)]
PREFILL_M = 512
W_SCALE = 0.02
METRIC = "1.58/1-bit linear: weight GB/s at M=1 & int8 TOPS at M=512, % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_DATASHEET_TOPS = 4500.0   # B200 dense int8 (datasheet; the 2:4-sparse figure is twice this)


def int8_peak(peaks):
    """int8 peak for a kernel timed in isolation: 2 x the measured burst bf16
    cuBLAS figure (the nominal int8/bf16 ratio of the tensor cores)."""
    return 2.0 * peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])


# DRAM bytes (read + write) per packed-weight byte of the chain kernel, from an
# ncu capture of a shorter chain of the same blocks (traffic grows with the
# weights streamed): the DRAM bytes read + written by one launch over the
# 2-block stack divided by its 101,187,584 weight bytes, cold caches.  None
# whenever the chain kernel has changed since the last capture.
CHAIN_TRAFFIC_PER_WEIGHT_BYTE = (101250560 + 3626496) / 101187584
CHAIN_TRAFFIC_SOURCE = ("ncu dram__bytes_read.sum + dram__bytes_write.sum of one chain_kernel<0> launch "
                        "over the 2-block stack (--layers 2, cold caches), scaled to this launch by its "
                        "weight bytes; summary under profiles/")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        d["_source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["_source"] = "fallback"
    return d


# ------------------------------------------------------------ clocks ------

class ClockSampler:
    """nvidia-smi sampling (200 ms) of SM clock and throttle reasons."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.t_start = self.t_stop = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self._reader = threading.Thread(target=self._read, daemon=True)
        self._reader.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, which):
        setattr(self, "t_" + which, time.time())

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((ts, float(parts[1]), float(parts[2]), parts))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0}
        inside = [r for r in rows if self.t_start and self.t_stop
                  and self.t_start - 0.1 <= r[0] <= self.t_stop + 0.1]
        window = "timed"
        if len(inside) < 1:
            inside, window = rows, "warmup+timed"
        mhz = sorted(r[1] for r in inside)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in inside:
            for i, n in enumerate(names):
                if r[3][5 + i].lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": mhz[len(mhz) // 2], "sm_max_mhz": inside[0][2],
                "reasons": sorted(reasons), "samples": len(inside), "window": window}


# ----------------------------------------------------------- workloads ----

def decode_stack(blw, synth, dev, form: str, M: int = 1, layers: int = LLAMA7B_LAYERS,
                 block=None):
    """Allocate and pack the 7B-shaped stack.  Every call's input and output are
    views into one contiguous device buffer each (so an end-to-end step is one
    host->device copy, the graph, and one device->host copy)."""
    block = block or LLAMA7B_BLOCK
    shapes = [(layer, j, K, N) for layer in range(layers) for j, (_, K, N) in enumerate(block)]
    x_all = torch.empty((sum(M * K for _, _, K, _ in shapes),), dtype=torch.float16, device=dev)
    y_all = torch.empty((sum(M * N for _, _, _, N in shapes),), dtype=torch.float16, device=dev)
    calls = []
    wbytes = 0
    xo = yo = 0
    for layer, j, K, N in shapes:
        seed = 2_000_000 + layer * 16 + j
        x = x_all[xo:xo + M * K].view(M, K)
        x.copy_(synth.activations(M, K, seed=seed, device=dev))
        y = y_all[yo:yo + M * N].view(M, N)
        xo += M * K
        yo += M * N
        if form == "ternary":
            w = synth.ternary_weights(N, K, seed=seed + 7, device=dev)
            packed = blw.bl_pack_ternary(w)
            del w
            ws = torch.empty((blw.bl_ternary_workspace_bytes(M, K, N),), dtype=torch.uint8, device=dev)
            calls.append(dict(x=x, w=packed, y=y, ws=ws, K=K, N=N))
        else:
            w = synth.sign_weights(N, K, seed=seed + 7, device=dev)
            packed = blw.ob_pack_sign(w)
            del w
            g = synth.value_vector(K, seed=seed + 8, device=dev)
            h = synth.value_vector(N, seed=seed + 9, device=dev)
            ws = torch.empty((blw.ob_workspace_bytes(M, K, N),), dtype=torch.uint8, device=dev)
            calls.append(dict(x=x, w=packed, y=y, ws=ws, g=g, h=h, K=K, N=N))
            wbytes += 2 * (K + N)
        wbytes += packed.numel() * 4
    torch.cuda.synchronize()
    return calls, wbytes, x_all, y_all


def run_calls(blw, calls, form):
    if form == "ternary":
        for c in calls:
            blw.bl_ternary_linear(c["x"], c["w"], W_SCALE, workspace=c["ws"], out=c["y"])
    else:
        for c in calls:
            blw.ob_linear(c["x"], c["w"], c["g"], c["h"], workspace=c["ws"], out=c["y"])


def block_sources(blocks: int):
    """Dependency pattern of a LLaMA-like decode step through the 7-layer block,
    each elementwise step between two linears taken as the identity: q, k, v
    read the block input (block 0: a given x; later: the previous block's down
    output), o reads v's output (attention's place), gate and up read o's
    output (the residual/norm's place), down reads gate's output (SwiGLU's)."""
    src = []
    for b in range(blocks):
        base = 7 * b
        blk_in = -1 if b == 0 else base - 1
        src += [blk_in, blk_in, blk_in, base + 2, base + 3, base + 3, base + 4]
    return src


def chain_stack(blw, synth, dev, form: str, dependent: bool, layers: int = LLAMA7B_LAYERS,
                fused: bool = False):
    """The 7B-shaped stack as decode-chain layers (M = 1).  dependent: the
    decode step's dependency pattern (one given input); else every layer reads
    its own given input.  fused (with dependent): q, k, v and gate, up read an
    RMSNorm of their input (one weight per block and place, counted in the
    weight bytes) and down reads SwiGLU(gate, up) -- the block's elementwise
    steps run inside the chain launch.  Returns (layer dicts, weight bytes, given-input
    buffer, output buffer); every layer's given x and y are views into those
    two buffers.  Ternary w_scale is 1/sqrt(2K/3) per layer, which keeps the
    activations O(1) along a dependent chain (timing does not depend on it)."""
    shapes = [(K, N) for _ in range(layers) for (_, K, N) in LLAMA7B_BLOCK]
    srcs = block_sources(layers) if dependent else [-1] * len(shapes)
    x_all = torch.empty((sum(K for (K, _), s in zip(shapes, srcs) if s < 0),), dtype=torch.float16,
                        device=dev)
    y_all = torch.empty((sum(N for _, N in shapes),), dtype=torch.float16, device=dev)
    out, wbytes, xo, yo = [], 0, 0, 0
    prev_x = None
    norm_w = None
    for j, ((K, N), s) in enumerate(zip(shapes, srcs)):
        seed = 2_000_000 + (j // 7) * 16 + j % 7
        d = dict(K=K, N=N, src=s, y=y_all[yo:yo + N])
        if fused and dependent:
            if j % 7 in (0, 4):            # attention and MLP RMSNorm weights of the block
                norm_w = synth.norm_weight(K, seed=seed + 10, device=dev)
                wbytes += 2 * K
            if j % 7 in (0, 1, 2, 4, 5):
                d["norm_w"], d["norm_eps"] = norm_w, 1e-5
            if j % 7 == 6:
                d["src2"] = j - 1          # down reads SwiGLU(gate, up), evaluated once per
                d["swiglu_buf"] = torch.empty((K,), dtype=torch.float16, device=dev)   # element
        yo += N
        if s < 0:
            if dependent and prev_x is not None and j % 7 in (1, 2):
                d["x"] = prev_x            # k and v read q's input
            else:
                d["x"] = x_all[xo:xo + K]
                d["x"].copy_(synth.activations(1, K, seed=seed, device=dev)[0])
                xo += K
            prev_x = d["x"]
        if form == "ternary":
            w = synth.ternary_weights(N, K, seed=seed + 7, device=dev)
            d["w"] = blw.bl_pack_ternary(w)
            d["w_scale"] = float(1.0 / (2.0 * K / 3.0) ** 0.5)
        else:
            w = synth.sign_weights(N, K, seed=seed + 7, device=dev)
            d["w"] = blw.ob_pack_sign(w)
            d["g"] = synth.value_vector(K, seed=seed + 8, device=dev)
            d["h"] = synth.value_vector(N, seed=seed + 9, device=dev)
            wbytes += 2 * (K + N)
        del w
        wbytes += d["w"].numel() * 4
        out.append(d)
    x_all = x_all[:xo]
    torch.cuda.synchronize()
    return out, wbytes, x_all, y_all


def capture(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm the path once outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def barrier(dist_on):
    if dist_on:
        torch.distributed.barrier()


def max_over_ranks(v: float, dist_on: bool, dev) -> float:
    """Slowest rank's time: every rank takes part, in the same order on all ranks."""
    if not dist_on:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: units all ranks processed / slowest rank's time (ms)."""
    return units_per_rank * world / (ms_max * 1e-3)


def time_replays(g, steps, warmup, dist_on, dev, clocks=None):
    for _ in range(warmup):
        g.replay()
    barrier(dist_on)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if clocks:
        clocks.mark("start")
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    if clocks:
        clocks.mark("stop")
    barrier(dist_on)
    ms = e0.elapsed_time(e1)
    return max_over_ranks(ms, dist_on, dev) / steps


# ------------------------------------------------------------- oracle -----

def oracle_decode_calls(synth, form: str, n_calls: int, parallel: bool = False,
                        budget_s: float = 1e9):
    """Time the oracle on calls of the decode stack (M=1), in stack order from
    its first call: at most n_calls calls and about budget_s seconds of oracle
    time.  Packing and input generation are outside the timed part.  Returns
    (packed-weight bytes, seconds, calls timed)."""
    import oracle
    oracle.build()
    total_bytes, t_total, calls = 0, 0.0, 0
    shapes = [(layer, j, K, N) for layer in range(LLAMA7B_LAYERS)
              for j, (_, K, N) in enumerate(LLAMA7B_BLOCK)]
    while calls < n_calls and t_total < budget_s:
        layer, j, K, N = shapes[calls % len(shapes)]
        seed = 2_000_000 + layer * 16 + j
        x = synth.activations(1, K, seed=seed).numpy()
        if form == "ternary":
            w2 = oracle.pack_ternary(synth.ternary_weights(N, K, seed=seed + 7).numpy())
            t0 = time.perf_counter()
            oracle.ternary_linear(x, w2, W_SCALE, parallel=parallel)
            t_total += time.perf_counter() - t0
            total_bytes += w2.nbytes
        else:
            s1 = oracle.pack_sign(synth.sign_weights(N, K, seed=seed + 7).numpy())
            g = synth.value_vector(K, seed=seed + 8).numpy()
            h = synth.value_vector(N, seed=seed + 9).numpy()
            t0 = time.perf_counter()
            oracle.ob_linear(x, s1, g, h, parallel=parallel)
            t_total += time.perf_counter() - t0
            total_bytes += s1.nbytes + 2 * (K + N)
        calls += 1
    return total_bytes, t_total, calls


def oracle_svid_seconds(synth):
    """The oracle's SVID (sign + rank-1 power iteration of |W|) of the OneBit
    workload's seeded 4096x4096 N(0, 0.02) matrix: (seconds, iterations)."""
    import oracle
    W = synth.svid_weights(4096, 4096, seed=1_000_001).numpy()
    t0 = time.perf_counter()
    *_, it = oracle.svid(W)
    return time.perf_counter() - t0, it


def cpu_baselines(synth):
    """The oracle timed on this host's cores: one core and all cores (OpenMP
    over output rows), each on a bounded sample of the decode stack (whole
    calls from its start, about 10 s each), plus the SVID oracle."""
    import oracle
    out = {}
    for key, parallel in (("all_cores", True), ("single_core", False)):
        b, t, n = oracle_decode_calls(synth, "ternary", 10 ** 9, parallel=parallel, budget_s=10.0)
        out[key] = {"value": round(b / t / 1e9, 4), "unit": "GB/s",
                    "cores": oracle.omp_threads() if parallel else 1, "kind": "oracle",
                    "sample": f"{n} calls of the stack (M=1) in stack order from its first call, "
                              f"{t:.1f} s of oracle time",
                    "seconds": round(t, 2)}
    secs, it = oracle_svid_seconds(synth)
    out["svid_4096x4096"] = {"seconds": round(secs, 2), "iterations": it, "cores": 1,
                             "kind": "oracle", "what": "sign + rank-1 power iteration of |W|, fp64"}
    return out


def run_case(blw, synth, dev, args, peaks):
    """Small named workloads for kernel profiles (one GPU):
    ternary_decode_m1   the ternary 7B-shaped stack at M = 1, one bl_ternary_linear
                        call per layer (args.layers blocks), as a CUDA graph;
    onebit_decode_m1    the same in OneBit form (ob_linear);
    onebit_prefill_m256 ob_linear at M = 256 on the 13B up (5120->13824) and down
                        (13824->5120) layers, as a CUDA graph."""
    if args.case in ("ternary_decode_m1", "onebit_decode_m1"):
        form = args.case.split("_")[0]
        calls, wbytes, _x, _y = decode_stack(blw, synth, dev, form, layers=args.layers)
        g = capture(lambda: run_calls(blw, calls, form))
        ms = time_replays(g, args.steps, args.warmup, False, dev)
        gbs = wbytes / (ms * 1e-3) / 1e9
        return {"ms_per_step": round(ms, 4), "weight_bytes_per_step": wbytes, "GBs": round(gbs, 1),
                "hbm_frac": round(gbs / peaks["hbm_gbs"], 4)}
    calls, ops = [], 0
    for j, (name, K, N) in enumerate(LLAMA13B_SWEEP):
        x = synth.activations(256, K, seed=5_000_000 + j, device=dev)
        w = synth.sign_weights(N, K, seed=5_000_010 + j, device=dev)
        calls.append(dict(x=x, w=blw.ob_pack_sign(w), g=synth.value_vector(K, seed=5_000_020 + j, device=dev),
                          h=synth.value_vector(N, seed=5_000_030 + j, device=dev),
                          y=torch.empty((256, N), dtype=torch.float16, device=dev),
                          ws=torch.empty((blw.ob_workspace_bytes(256, K, N),), dtype=torch.uint8, device=dev)))
        del w
        ops += 2 * 256 * K * N
    g = capture(lambda: run_calls(blw, calls, "onebit"))
    ms = time_replays(g, args.steps, args.warmup, False, dev)
    return {"ms_per_step": round(ms, 4), "int8_equiv_TOPS": round(ops / (ms * 1e-3) / 1e12, 2),
            "shapes_KxN": [[K, N] for (_, K, N) in LLAMA13B_SWEEP]}


def run_prefill(blw, synth, dev, args, dist_on, world, peaks):
    """M=512 on the LLaMA-70B-shaped ternary layers (tcgen05 prefill path)."""
    pcalls = []
    flops = 0
    for j, (name, K, N) in enumerate(LLAMA70B_PREFILL):
        seed = 3_000_000 + j
        x = synth.activations(PREFILL_M, K, seed=seed, device=dev, outlier_frac=0.01)
        w = synth.ternary_weights(N, K, seed=seed + 7, device=dev)
        w2 = blw.bl_pack_ternary(w)
        del w
        ws = torch.empty((blw.bl_ternary_workspace_bytes(PREFILL_M, K, N),), dtype=torch.uint8,
                         device=dev)
        pcalls.append(dict(x=x, w=w2, y=torch.empty((PREFILL_M, N), dtype=torch.float16,
                                                   device=dev), ws=ws, K=K, N=N))
        flops += 2 * PREFILL_M * K * N
    pg = capture(lambda: run_calls(blw, pcalls, "ternary"))
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    # enough replays that the 200 ms clock sampler sees the timed region (~1.5 s)
    est = time_replays(pg, 20, args.warmup, dist_on, dev)
    pms = time_replays(pg, max(args.steps, int(1500.0 / max(est, 1e-3))), 3, dist_on, dev, clocks)
    time.sleep(0.3)
    clocks.stop()
    tops = flops * world / (pms * 1e-3) / 1e12
    i8_peak = int8_peak(peaks)
    del pg, pcalls
    torch.cuda.synchronize()
    return {
        "workload": "llama70b-prefill-M512-ternary (8192x8192, 8192x28672, 28672x8192; 1% outlier channels x20)",
        "value": round(tops, 2), "unit": "TOPS", "ms_per_step": round(pms, 4),
        "roofline": {"bound": "tensor", "achieved": round(tops / world, 2), "peak": round(i8_peak, 1),
                     "unit": "TOPS", "frac": round(tops / world / i8_peak, 4),
                     "peak_source": "2 x measured burst bf16 cuBLAS (nominal int8/bf16 ratio); "
                                    "the step is timed alone",
                     "frac_of_datasheet_4500": round(tops / world / INT8_DATASHEET_TOPS, 4)},
        "clocks": clocks.summary()}


def run_sweep(blw, synth, dev, peaks, reps=10, forms=("ternary", "onebit"), layers=None,
              ms_list=None):
    """Per (form, layer, M): the effective weight GB/s and int8 TOPS of one call,
    over rotating weight copies that total more than twice the L2 (each call
    streams its weights from HBM).  Defaults: the LLaMA-13B-shaped batch sweep."""
    l2_bytes = 126 * 2 ** 20
    i8_peak = int8_peak(peaks)
    layers = layers or LLAMA13B_SWEEP
    ms_list = ms_list or SWEEP_M
    out = []
    for form in forms:
        for (name, K, N) in layers:
            planes = 2 if form == "billm" else 1        # BiLLM: two stacked sign planes
            wb = planes * N * K // (4 if form == "ternary" else 8)
            copies = max(2, -(-2 * l2_bytes // wb) + 1)
            ws, gs, hs = [], None, None
            for c in range(copies):
                seed = 4_000_000 + 100 * c + (0 if name == "up" else 50)
                if form == "ternary":
                    w = synth.ternary_weights(N, K, seed=seed, device=dev)
                    ws.append(blw.bl_pack_ternary(w))
                else:
                    w = synth.sign_weights(planes * N, K, seed=seed, device=dev)
                    ws.append(blw.ob_pack_sign(w))
                del w
            if form == "onebit":
                gs = synth.value_vector(K, seed=4_000_900, device=dev)
                hs = synth.value_vector(N, seed=4_000_901, device=dev)
            if form == "billm":
                hs = synth.value_vector(2 * N, seed=4_000_902, device=dev)    # alpha_o, alpha_r
            for M in ms_list:
                x = synth.activations(M, K, seed=4_001_000 + M, device=dev)
                y = torch.empty((M, N), dtype=torch.float16, device=dev)
                nws = {"ternary": blw.bl_ternary_workspace_bytes, "onebit": blw.ob_workspace_bytes,
                       "billm": blw.billm_workspace_bytes}[form](M, K, N)
                wsp = torch.empty((nws,), dtype=torch.uint8, device=dev)

                def step():
                    for w2 in ws:
                        if form == "ternary":
                            blw.bl_ternary_linear(x, w2, W_SCALE, workspace=wsp, out=y)
                        elif form == "billm":
                            blw.billm_linear(x, w2, hs, workspace=wsp, out=y)
                        else:
                            blw.ob_linear(x, w2, gs, hs, workspace=wsp, out=y)

                g = capture(step)
                ms = time_replays(g, reps, 3, False, dev) / copies
                vec = {"ternary": 0, "onebit": 2 * (K + N), "billm": 4 * N}[form]
                gbs = (wb + vec) / (ms * 1e-3) / 1e9
                tops = 2 * planes * M * K * N / (ms * 1e-3) / 1e12
                out.append({"form": form, "layer": f"{name} {K}->{N}", "M": M, "us_per_call": round(ms * 1e3, 2),
                            "weight_GBs": round(gbs, 1), "TOPS": round(tops, 2),
                            "hbm_frac": round(gbs / peaks["hbm_gbs"], 4),
                            "int8_frac": round(tops / i8_peak, 4)})
                del g, x, y, wsp
            del ws
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
    return out


# --------------------------------------------------------------- main -----

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--no-extras", action="store_true", help="headline workload only")
    ap.add_argument("--layers", type=int, default=LLAMA7B_LAYERS,
                    help="blocks in the decode stack (fewer = a small profiling case)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="skip the 13B batch sweep")
    ap.add_argument("--case", default=None,
                    choices=["ternary_decode_m1", "onebit_decode_m1", "onebit_prefill_m256"],
                    help="time one small named workload (for profiling) and print its line only")
    ap.add_argument("--prefill-only", action="store_true",
                    help="run only the M=512 prefill layers (a profiling case)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    from bit_weight_linear_b200 import synth

    if args.impl == "reference":
        # The oracle (scalar C on the host cores) is this workload's reference
        # arm.  A whole 224-call step takes it minutes, so each of its steps is
        # one call of the stack, in stack order (warm-up calls first); value is
        # the packed-weight GB/s over exactly the calls timed.
        if rank != 0:
            return 0
        import oracle
        oracle_decode_calls(synth, "ternary", args.warmup, parallel=True)
        b, secs, n = oracle_decode_calls(synth, "ternary", args.steps, parallel=True,
                                         budget_s=120.0)
        gbs = b / secs / 1e9
        line = {"impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
                "n_gpus": args.gpus, "steps": n, "warmup": args.warmup,
                "ms_per_step": round(secs / n * 1e3, 3), "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "s8", "data": "synthetic",
                "config": {"workload": "llama7b-decode-M1-ternary-bitlinear-32x7",
                           "M": 1, "layers": LLAMA7B_LAYERS, "parallelism": "replicas",
                           "step": "one linear call of the 224-call stack, in stack order"},
                "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s",
                                 "cores": oracle.omp_threads(), "kind": "oracle",
                                 "sample": f"{n} calls from the start of the stack (M=1), "
                                           f"{secs:.1f} s of oracle time"},
                "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_on = world > 1
    if dist_on:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)

    import bit_weight_linear_b200 as blw
    from bit_weight_linear_b200 import build
    build.build()
    peaks = load_peaks()

    if args.case:
        res = run_case(blw, synth, dev, args, peaks)
        if rank == 0:
            print(json.dumps({"case": args.case, **res}), flush=True)
        if dist_on:
            torch.distributed.destroy_process_group()
        return 0

    if args.prefill_only:
        res = run_prefill(blw, synth, dev, args, dist_on, world, peaks)
        if rank == 0:
            print(json.dumps({"prefill": res}), flush=True)
        if dist_on:
            torch.distributed.destroy_process_group()
        return 0

    # ---- headline: the ternary 7B-shaped stack at M = 1 as ONE decode-chain launch per step,
    # with a decode step's dependency pattern
    chain_layers, wbytes, x_all, y_all = chain_stack(blw, synth, dev, "ternary", dependent=True,
                                                     layers=args.layers)
    in_b, out_b = x_all.numel() * 2, y_all.numel() * 2
    chain = blw.Chain(0, chain_layers)
    g = capture(chain.run)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ms = time_replays(g, args.steps, args.warmup, dist_on, dev, clocks)
    time.sleep(0.3)
    clocks.stop()
    n_layers = len(chain_layers)
    value = whole_job_rate(wbytes, world, ms) / 1e9

    # roofline of the one kernel of the step: the persistent chain kernel
    alg_bytes = wbytes + in_b + out_b
    achieved = alg_bytes / (ms * 1e-3) / 1e9
    roofline = {"kernel": "chain_kernel<0> (one persistent launch per step; all 224 layers)",
                "bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "algorithmic_bytes_per_launch": alg_bytes,
                "traffic": round(CHAIN_TRAFFIC_PER_WEIGHT_BYTE * wbytes) if CHAIN_TRAFFIC_PER_WEIGHT_BYTE else None,
                "traffic_unit": "bytes",
                "traffic_source": CHAIN_TRAFFIC_SOURCE,
                "peak_source": peaks["_source"],
                "note": "launch duration = timed region / steps (one chain kernel and one "
                        f"{4 * n_layers}-byte counter memset per step)"}

    # ---- e2e: host buffers through the C ABI.  Every step is one bl_chain_run_host call: the
    # step's given input copied from pinned host memory, the chain, and every layer's output
    # copied back, all inside the timed region.  Two chains over two device buffer sets run on two
    # streams in turn, so one step's copies overlap the neighbouring step's kernel.
    xin = x_all.cpu().pin_memory()
    youts = [torch.empty(y_all.shape, dtype=torch.float16).pin_memory() for _ in range(2)]
    x_all2, y_all2 = torch.empty_like(x_all), torch.empty_like(y_all)

    def rebased(t, base, other):
        off = t.storage_offset() - base.storage_offset()
        return other[off:off + t.numel()].view(t.shape)

    layers2 = [dict(d, y=rebased(d["y"], y_all, y_all2),
                    **({"x": rebased(d["x"], x_all, x_all2)} if "x" in d else {})) for d in chain_layers]
    chain2 = blw.Chain(0, layers2)
    sets = [(chain, x_all, y_all), (chain2, x_all2, y_all2)]
    comp = torch.cuda.current_stream()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]

    def e2e_run(n):
        for st in streams:
            st.wait_stream(comp)
        for i in range(n):
            ch, xs, ys = sets[i % 2]
            with torch.cuda.stream(streams[i % 2]):
                ch.run_host([(xin, xs)], [(ys, youts[i % 2])])
        for st in streams:
            comp.wait_stream(st)

    e2e_run(args.warmup)
    barrier(dist_on)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e2e_steps = max(10, args.steps // 4)
    e0.record(comp)
    e2e_run(e2e_steps)
    e1.record(comp)
    torch.cuda.synchronize()
    barrier(dist_on)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist_on, dev) / e2e_steps
    assert blw.bl_device_status() == 0, "a bounded wait expired in the chain kernel"
    assert torch.equal(youts[(e2e_steps - 1) % 2], y_all.cpu()), "e2e outputs differ from the device run"
    e2e = {"value": round(wbytes * world / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
           "h2d_bytes_per_step": xin.numel() * 2, "d2h_bytes_per_step": youts[0].numel() * 2,
           "ms_per_step": round(e2e_ms, 4),
           "call": "bl_chain_run_host (host buffers; one H2D copy, the chain, one D2H copy per step)",
           "overlap": "two chains on two streams in turn: one step's copies overlap the other's kernel"}
    del sets, streams, chain2, layers2, x_all2, y_all2
    del g, chain, chain_layers, x_all, y_all
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    extras = {}
    if not args.no_extras:
        # ---- the same stack as one chain launch whose layers all read their own given input
        ilayers, iwbytes, _ix, _iy = chain_stack(blw, synth, dev, "ternary", dependent=False,
                                                 layers=args.layers)
        ich = blw.Chain(0, ilayers)
        ig = capture(ich.run)
        ims = time_replays(ig, args.steps, args.warmup, dist_on, dev)
        ival = iwbytes * world / (ims * 1e-3) / 1e9
        extras["decode_chain_independent"] = {
            "workload": "llama7b-decode-M1-ternary-32x7, one chain launch, every layer its own input",
            "value": round(ival, 2), "unit": "GB/s", "ms_per_step": round(ims, 4),
            "roofline": {"bound": "hbm", "achieved": round(ival / world, 1), "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": round(ival / world / peaks["hbm_gbs"], 4)}}
        del ig, ich, ilayers, _ix, _iy
        torch.cuda.synchronize()
        torch.cuda.empty_cache()

        # ---- the dependent step with RMSNorm and SwiGLU fused into the chain
        flayers, fwbytes, _fx, _fy = chain_stack(blw, synth, dev, "ternary", dependent=True,
                                                 layers=args.layers, fused=True)
        fch = blw.Chain(0, flayers)
        fg = capture(fch.run)
        fms = time_replays(fg, args.steps, args.warmup, dist_on, dev)
        assert blw.bl_device_status() == 0, "a bounded wait expired in the chain kernel"
        fval = fwbytes * world / (fms * 1e-3) / 1e9
        extras["decode_chain_fused"] = {
            "workload": "llama7b-decode-M1-ternary-32x7, one chain launch, decode-step dependencies, "
                        "RMSNorm (q,k,v; gate,up) and SwiGLU (down) fused",
            "value": round(fval, 2), "unit": "GB/s", "ms_per_step": round(fms, 4),
            "weight_bytes_per_step": fwbytes,
            "roofline": {"bound": "hbm", "achieved": round(fval / world, 1), "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": round(fval / world / peaks["hbm_gbs"], 4)}}
        del fg, fch, flayers, _fx, _fy
        torch.cuda.synchronize()
        torch.cuda.empty_cache()

        # ---- OneBit: the same dependent decode-chain step
        olayers, owbytes, _ox, _oy = chain_stack(blw, synth, dev, "onebit", dependent=True,
                                                 layers=args.layers)
        och = blw.Chain(1, olayers)
        og = capture(och.run)
        oms = time_replays(og, args.steps, args.warmup, dist_on, dev)
        oval = owbytes * world / (oms * 1e-3) / 1e9
        extras["onebit_decode"] = {
            "workload": "llama7b-decode-M1-onebit-32x7, one chain launch, decode-step dependencies",
            "value": round(oval, 2), "unit": "GB/s", "ms_per_step": round(oms, 4),
            "weight_bytes_per_step": owbytes,
            "roofline": {"bound": "hbm", "achieved": round(oval / world, 1), "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": round(oval / world / peaks["hbm_gbs"], 4)}}
        del og, och, olayers, _ox, _oy
        torch.cuda.synchronize()
        torch.cuda.empty_cache()

        # ---- SVID initialisation of the OneBit 4096x4096 layer on the device
        W = synth.svid_weights(4096, 4096, seed=1_000_001, device=dev)
        for _ in range(3):
            blw.ob_svid(W)
        sv_ms = []
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            _s1, _g, _h, sv_sigma, sv_it = blw.ob_svid(W)
            e1.record()
            torch.cuda.synchronize()
            sv_ms.append(e0.elapsed_time(e1))
        sv_med = sorted(sv_ms)[len(sv_ms) // 2]
        sv_passes = 1 + 2 * sv_it                   # sign pass + a row and a column pass per iteration
        extras["svid_4096x4096"] = {
            "workload": "ob_svid of a 4096x4096 N(0, 0.02) fp32 W (sign pack + rank-1 power iteration "
                        "of |W| in fp64, tol 1e-12)",
            "ms": round(sv_med, 4), "iterations": sv_it, "sigma": sv_sigma,
            "w_passes": sv_passes,
            "w_GBs": round(sv_passes * W.numel() * 4 / (sv_med * 1e-3) / 1e9, 1),
            "note": "includes the call's host read-backs of the convergence flag; W (64 MB) stays in L2"}
        del W, _s1, _g, _h
        torch.cuda.synchronize()

        # ---- the per-call path: 224 bl_ternary_linear / ob_linear calls per step in a graph
        for form in ("ternary", "onebit"):
            pcalls, pwbytes, _px, _py = decode_stack(blw, synth, dev, form, layers=args.layers)
            pg = capture(lambda: run_calls(blw, pcalls, form))
            pms = time_replays(pg, max(10, args.steps // 2), args.warmup, dist_on, dev)
            pval = pwbytes * world / (pms * 1e-3) / 1e9
            extras[f"decode_per_call_{form}"] = {
                "workload": f"llama7b-decode-M1-{form}-32x7, one library call per layer (CUDA graph)",
                "value": round(pval, 2), "unit": "GB/s", "ms_per_step": round(pms, 4),
                "roofline": {"bound": "hbm", "achieved": round(pval / world, 1),
                             "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": round(pval / world / peaks["hbm_gbs"], 4)}}
            del pg, pcalls, _px, _py
            torch.cuda.synchronize()
            torch.cuda.empty_cache()

        extras["prefill"] = run_prefill(blw, synth, dev, args, dist_on, world, peaks)
        # the two small configurations: BitLinear M=8 and OneBit M=1 / M=16 on 4096x4096
        extras["bitlinear_m8_4096"] = run_sweep(blw, synth, dev, peaks, forms=("ternary",),
                                                layers=[("q", 4096, 4096)], ms_list=[8])
        extras["onebit_4096"] = run_sweep(blw, synth, dev, peaks, forms=("onebit",),
                                          layers=[("q", 4096, 4096)], ms_list=[1, 16])
        # the two-plane binary layer (BiLLM residual approximation) on the same shapes
        extras["billm_4096"] = run_sweep(blw, synth, dev, peaks, forms=("billm",),
                                         layers=[("q", 4096, 4096), ("up", 4096, 11008)],
                                         ms_list=[1, 16, 256])
        # the decode sweep per layer shape: each 7B-shaped layer alone at M=1, in a
        # chain of calls over rotating weight copies larger than L2
        extras["decode_layers_7b"] = run_sweep(blw, synth, dev, peaks, forms=("ternary", "onebit"),
                                               layers=[("q/k/v/o", 4096, 4096), ("gate/up", 4096, 11008),
                                                       ("down", 11008, 4096)], ms_list=[1])
        if not args.no_sweep:
            extras["batch_sweep_13b"] = run_sweep(blw, synth, dev, peaks)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "s8",
        "data": "synthetic",
        "config": {"workload": "llama7b-decode-M1-ternary-bitlinear-32x7", "M": 1,
                   "layers": args.layers, "shapes_KxN": [[K, N] for _, K, N in LLAMA7B_BLOCK],
                   "weight_bytes_per_step": wbytes, "w_scale": "1/sqrt(2K/3) per layer",
                   "dependencies": "decode step: q,k,v <- block input; o <- v; gate,up <- o; "
                                   "down <- gate; next block input <- down",
                   "l2": "inputs larger than L2 (1.62 GB packed weights per step, 126 MB L2)",
                   "parallelism": f"replicas x{world}",
                   "graph": "CUDA graph of one bl_chain_run (counter memset + one kernel)"},
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clocks.summary(),
    }
    line.update(extras)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baselines(synth)
        line["cpu_baseline"] = dict(cb["all_cores"], single_core=cb["single_core"],
                                    svid_4096x4096=cb["svid_4096x4096"])
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
