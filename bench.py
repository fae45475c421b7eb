#!/usr/bin/env python
"""Benchmark: QLoRA NF4 linear layer with LoRA on B200.

One step = one pass of the whole hot path over one batch of the 65B-shaped
transformer block (hidden 8192; q, k, v, o 8192x8192, gate/up 8192->22016, down
22016->8192; 4096 tokens; LoRA r=64, alpha=16 on every layer): for each layer
quantise its bf16 weight to NF4 with double-quantised scales, run the forward
(T = X A^T; Y = X W'^T + s T B^T), then run the backward of every layer in
reverse order (dX, dA, dB).  value = algorithmic forward+backward FLOPs
(4MNK + 6Mr(N+K) per layer) / device time of the step.

Launch:  python bench.py [--gpus N --steps K --warmup W] [--impl reference]
N > 1 runs under torch.distributed (one process per GPU, NCCL): every rank runs
its own 4096 tokens through the same frozen weights (weak scaling) and the LoRA
gradients dA, dB of all layers are summed across ranks with one all-reduce per
step (data parallelism's only exchange).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QLoRA NF4 linear fwd+bwd TFLOP/s; NF4 GEMV GB/s; % of roofline (1×B200)"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# DRAM bytes (read + write) of one fused forward GEMM launch, mean over the block's
# seven layers (4 of 8192x8192, 2 of 22016x8192, 1 of 8192x22016), from ncu
# captures of the `cases` module's fwd_8192 / fwd_65b_up / fwd_65b_down.  The
# figure belongs to the kernel sources it was measured on: it is reported only
# while their digest still matches, else the traffic is null.
FUSED_FWD_TRAFFIC_BYTES = 592.60e6
FUSED_FWD_TRAFFIC_SOURCES = ("gemm_pair_kernel.cuh", "gemm_kernel.cuh", "sm100_ptx.cuh", "nf4_device.cuh",
                             "qlora_nf4.cu")
FUSED_FWD_TRAFFIC_DIGEST = "aa961c27569a8b40"


def fused_fwd_traffic():
    import hashlib

    h = hashlib.sha256()
    for f in FUSED_FWD_TRAFFIC_SOURCES:
        with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "bit_nf4_quantized_27_b200", "csrc", f),
                  "rb") as fh:
            h.update(fh.read())
    return FUSED_FWD_TRAFFIC_BYTES if h.hexdigest()[:16] == FUSED_FWD_TRAFFIC_DIGEST else None


def layer_flops(m, n, k, r):
    fwd = 2 * m * n * k + 2 * m * r * (k + n)
    bwd = 2 * m * n * k + 4 * m * r * (n + k)
    return fwd, bwd


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.dev)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample of the same step)
# ---------------------------------------------------------------------------
def oracle_sample(seconds_budget=20.0, rows=2048, toks=1024, wl=None):
    """Runs the oracle on row/token slices of a block's layers (the 65B-shaped
    block unless `wl` names another): quantise a `rows`-row slice of each weight,
    then forward+backward of `toks` tokens through it, layer after layer until
    `seconds_budget` is spent.  Returns (TFLOP/s, threads, description, seconds)."""
    import numpy as np
    from threadpoolctl import threadpool_info

    import oracle as O
    from bit_nf4_quantized_27_b200 import inputs as I

    wl = I.L65B_BLOCK if wl is None else wl
    flops, t_total, done = 0.0, 0.0, []
    for li, ly in enumerate(wl.layers):
        w = I.normal((rows, ly.k), 0.02, I.seed_for(wl.wid, I.W_ID, li)).float().numpy()
        x = I.normal((toks, ly.k), 1.0, I.seed_for(wl.wid, I.X_ID, li)).float().numpy()
        a = I.normal((wl.r, ly.k), ly.k ** -0.5, I.seed_for(wl.wid, I.A_ID, li)).float().numpy()
        b = I.normal((rows, wl.r), 0.01, I.seed_for(wl.wid, I.B_ID, li)).float().numpy()
        dy = I.normal((toks, rows), 1.0, I.seed_for(wl.wid, I.DY_ID, li)).float().numpy()
        t0 = time.perf_counter()
        q = O.quantize(w, rows, ly.k)
        wd = O.dequantize(q["codes"], q["scale_codes"], q["c2"], rows, ly.k)
        y, t = O.linear_fwd(wd, a, b, x, wl.alpha, wl.r)
        O.linear_bwd(wd, a, b, x, dy, wl.alpha, wl.r, t)
        t_total += time.perf_counter() - t0
        f, g = layer_flops(toks, rows, ly.k, wl.r)
        flops += f + g
        done.append(ly.name)
        if t_total > seconds_budget:
            break
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    desc = (f"oracle (numpy float64) on layers {','.join(done)} of {wl.name}, each a {rows}-row slice of W "
            f"quantised then forward+backward of {toks} tokens; FLOPs counted as for the GPU step")
    return flops / t_total / 1e12, threads, desc, t_total


def run_reference(args, rank):
    """The oracle, as it stands, on the host cores (bounded samples per step)."""
    if rank != 0:
        return
    vals = []
    for i in range(args.warmup + args.steps):
        v, threads, desc, secs = oracle_sample(seconds_budget=args.ref_seconds, rows=512, toks=512)
        if i >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    from bit_nf4_quantized_27_b200 import inputs as I

    wl = I.L65B_BLOCK
    step_flops = sum(sum(layer_flops(wl.m, ly.n, ly.k, wl.r)) for ly in wl.layers)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            # one full step of the workload at the sample's measured rate
            "ms_per_step": step_flops / (value * 1e12) * 1e3, "ms_per_step_kind": "extrapolated from the sample",
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config():
    return {"workload": "65b_block_m4096_r64", "hidden": 8192, "intermediate": 22016, "tokens_per_gpu": 4096,
            "layers": ["q", "k", "v", "o", "gate", "up", "down"], "lora_r": 64, "lora_alpha": 16,
            "step": "per layer: quantise bf16 W -> NF4 (+E4M3 scales), forward; then backward of all layers",
            "l2": "inputs larger than L2 (about 4.5 GB touched per step)", "parallelism": "dp"}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def cuda_timer():
    import torch

    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


def build_block(wl, device, rank, gen_seed_offset=0):
    """Device-resident inputs for every layer (drawn on the device with the
    per-tensor seeds of the input recipe; rank offsets the activation seeds)."""
    import torch

    from bit_nf4_quantized_27_b200 import binding as bd
    from bit_nf4_quantized_27_b200 import dp
    from bit_nf4_quantized_27_b200 import inputs as I

    def dnormal(shape, std, seed):
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        return (torch.randn(*shape, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)

    layers = []
    m, r = wl.m, wl.r
    for li, ly in enumerate(wl.layers):
        d = {"n": ly.n, "k": ly.k, "name": ly.name}
        d["w"] = dnormal((ly.n, ly.k), 0.02, I.seed_for(wl.wid, I.W_ID, li))
        d["a"] = dnormal((r, ly.k), ly.k ** -0.5, I.seed_for(wl.wid, I.A_ID, li))
        d["b"] = dnormal((ly.n, r), 0.01, I.seed_for(wl.wid, I.B_ID, li))
        d["x"] = dnormal((m, ly.k), 1.0, I.seed_for(wl.wid, I.X_ID, li) + 1000003 * rank)
        d["dy"] = dnormal((m, ly.n), 1.0, I.seed_for(wl.wid, I.DY_ID, li) + 1000003 * rank)
        d["q"] = bd.NF4Weight(ly.n, ly.k, device)
        d["y"] = torch.empty(m, ly.n, dtype=torch.bfloat16, device=device)
        d["t"] = torch.empty(2, m, r, dtype=torch.bfloat16, device=device)
        d["dx"] = torch.empty(m, ly.k, dtype=torch.bfloat16, device=device)
        d["ws_f"] = bd.new_workspace(bd.workspace_bytes(m, ly.n, ly.k, r, False), device)
        d["ws_b"] = bd.new_workspace(bd.workspace_bytes(m, ly.n, ly.k, r, True), device)
        layers.append(d)
    # one flat fp32 buffer holds every layer's dA and dB (one all-reduce per step)
    shapes = [(d["n"], d["k"]) for d in layers]
    flat = torch.zeros(dp.flat_size(shapes, r), dtype=torch.float32, device=device)
    for d, (da, db) in zip(layers, dp.grad_views(flat, shapes, r)):
        d["da"], d["db"] = da, db
    return layers, flat


def run_step(layers, wl, flat, world, timing=None, ready=None, quant=True):
    """One block step on the current stream.  `ready` = (x_events, dy_events):
    layer i's forward waits for x_events[i] and its backward for dy_events[i]
    (the end-to-end step copies each layer's inputs on a copy stream).  With
    quant=False the weights quantised by an earlier step are reused (the
    training step proper: QLoRA quantises the frozen weights once, at load)."""
    import torch

    from bit_nf4_quantized_27_b200 import binding as bd

    ev = timing is not None
    cur = torch.cuda.current_stream()
    for i, d in enumerate(layers):
        if ev:
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            e0.record()
        if quant:
            bd.quantize(d["w"], out=d["q"], ws=d["ws_f"])
        if ev:
            e1.record()
        if ready is not None:
            cur.wait_event(ready[0][i])
        bd.linear_fwd(d["q"], d["a"], d["b"], wl.alpha, d["x"], ws=d["ws_f"], out=d["y"], t_out=d["t"])
        if ev:
            e2.record()
            timing["quant"].append((e0, e1))
            timing["fwd"].append((e1, e2))
    for i in reversed(range(len(layers))):
        d = layers[i]
        if ev:
            e0, e1 = (torch.cuda.Event(enable_timing=True) for _ in range(2))
            e0.record()
        if ready is not None:
            cur.wait_event(ready[1][i])
        bd.linear_bwd(d["q"], d["a"], d["b"], wl.alpha, d["x"], d["dy"], d["t"], ws=d["ws_b"],
                      outs=(d["dx"], d["da"], d["db"]), grad_dtype=torch.float32)
        if ev:
            e1.record()
            timing["bwd"].append((e0, e1))
    if world > 1:
        from bit_nf4_quantized_27_b200 import dp

        dp.allreduce_grads(flat)


def launches_per_step(nlayers):
    # per layer of the 65B-shaped block: quantise 1; forward 3 (T with split K and
    # its finishing sum, fused GEMM); backward 4 (U with split K and its finishing
    # sum, dX, dA and dB in one launch) -- 56 per step, as the ncu launch list of
    # the step shows
    return nlayers * 8


def graph_time_us(calls, reps=5):
    """Captures `calls()` (a sequence of enqueues) into a CUDA graph and returns
    the device time of one replay in microseconds (CUDA events, median of reps).
    Graph replay removes the host enqueue cost, which exceeds the kernel time of
    a microsecond-scale call."""
    import torch

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        calls()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        calls()
    g.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        s, e = cuda_timer()
        s.record()
        g.replay()
        e.record()
        torch.cuda.synchronize()
        times.append(s.elapsed_time(e) * 1e3)
    del g
    return statistics.median(times)


def sub_gemv(device, peaks):
    """Decode-shaped forward (W 11008x4096, M in {1,4,16}, r=64): GB/s over the
    NF4 codes + scales + activations.  68 calls per CUDA graph, rotating over 17
    weight copies (395 MB, more than three times L2), so every call reads its
    weights from HBM."""
    import torch

    from bit_nf4_quantized_27_b200 import binding as bd
    from bit_nf4_quantized_27_b200 import inputs as I

    wl = I.GEMV
    n, k, r = 11008, 4096, 64
    copies = 17
    g = torch.Generator(device=device)
    g.manual_seed(I.seed_for(wl.wid, I.W_ID))
    qs = []
    for c in range(copies):
        w = (torch.randn(n, k, generator=g, device=device) * 0.02).to(torch.bfloat16)
        qs.append(bd.quantize(w))
        del w
    a = (torch.randn(r, k, generator=g, device=device) / 64).to(torch.bfloat16)
    b = (torch.randn(n, r, generator=g, device=device) * 0.01).to(torch.bfloat16)
    out = {}
    for m in (1, 4, 16):
        x = torch.randn(m, k, generator=g, device=device).to(torch.bfloat16)
        y = torch.empty(m, n, dtype=torch.bfloat16, device=device)
        t = torch.empty(2, m, r, dtype=torch.bfloat16, device=device)
        ws = bd.new_workspace(bd.workspace_bytes(m, n, k, r, False), device)
        reps = 4 * copies

        def calls():
            for i in range(reps):
                bd.linear_fwd(qs[i % copies], a, b, wl.alpha, x, ws=ws, out=y, t_out=t)

        us = graph_time_us(calls) / reps
        nf4 = n * k // 2 + n * k // 64 + 4 * ((n * k // 64 + 255) // 256)
        act = m * k * 2 + m * n * 2
        gbs = (nf4 + act) / (us * 1e-6) / 1e9
        out[f"m{m}"] = {"us_per_call": us, "GB/s": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"],
                        "GB/s_incl_adapters": (nf4 + act + (r * k + n * r) * 2) / (us * 1e-6) / 1e9,
                        "launches_per_call": 1, "timing": f"CUDA graph of {reps} calls, {copies} weight copies"}
    # 16 decode tokens, each with its own adapter on the same base
    m = 16
    ads = [((torch.randn(r, k, generator=g, device=device) / 64).to(torch.bfloat16),
            (torch.randn(n, r, generator=g, device=device) * 0.01).to(torch.bfloat16), wl.alpha) for _ in range(m)]
    x = torch.randn(m, k, generator=g, device=device).to(torch.bfloat16)
    y = torch.empty(m, n, dtype=torch.bfloat16, device=device)
    ws = bd.new_workspace(bd.workspace_bytes_multi(m, n, k, r), device)
    reps = 4 * copies
    idx = list(range(m))

    def calls_multi():
        for i in range(reps):
            bd.linear_fwd_multi(qs[i % copies], ads, idx, x, ws=ws, out=y)

    us = graph_time_us(calls_multi) / reps
    nf4 = n * k // 2 + n * k // 64 + 4 * ((n * k // 64 + 255) // 256)
    act = m * k * 2 + m * n * 2
    gbs = (nf4 + act) / (us * 1e-6) / 1e9
    out["m16_16_adapters"] = {"us_per_call": us, "GB/s": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"],
                              "GB/s_incl_adapters": (nf4 + act + m * (r * k + n * r) * 2) / (us * 1e-6) / 1e9,
                              "launches_per_call": 2, "timing": f"CUDA graph of {reps} calls, {copies} weight copies"}
    return out


def sub_block7b(device, peaks, steps=10, warmup=3):
    """The Llama-7B block (q, k, v, o 4096x4096, gate/up 4096->11008, down
    11008->4096; 2048 tokens, r = 64 on every layer): forward + backward of all
    seven layers, with the per-step quantisation and without it (the training
    step proper, weights quantised once at load); TFLOP/s of algorithmic FLOPs
    against the bf16 dense peak, and the oracle timed on a bounded sample of
    the same layers.  Inputs total about 1 GB, larger than L2."""
    import torch

    from bit_nf4_quantized_27_b200 import inputs as I

    wl = I.LLAMA7B_BLOCK
    layers, flat = build_block(wl, device, 0)
    fl_f = sum(layer_flops(wl.m, d["n"], d["k"], wl.r)[0] for d in layers)
    fl_b = sum(layer_flops(wl.m, d["n"], d["k"], wl.r)[1] for d in layers)
    for _ in range(warmup):
        run_step(layers, wl, flat, 1)
    torch.cuda.synchronize()
    res = {"flops_per_step": fl_f + fl_b, "layers": [d["name"] for d in layers], "tokens": wl.m, "lora_r": wl.r}
    for quant in (True, False):
        timing = {"quant": [], "fwd": [], "bwd": []}
        s, e = cuda_timer()
        s.record()
        for _ in range(steps):
            run_step(layers, wl, flat, 1, timing, quant=quant)
        e.record()
        torch.cuda.synchronize()
        ms = s.elapsed_time(e) / steps
        t_fwd = sum(a.elapsed_time(b) for a, b in timing["fwd"]) / steps
        t_bwd = sum(a.elapsed_time(b) for a, b in timing["bwd"]) / steps
        tag = "" if quant else "_no_quant"
        res["ms_per_step" + tag] = ms
        res["TFLOP/s" + tag] = (fl_f + fl_b) / (ms * 1e-3) / 1e12
        res["frac_of_bf16" + tag] = res["TFLOP/s" + tag] / peaks["bf16_tflops"]
        if quant:
            res["quantize_ms"] = sum(a.elapsed_time(b) for a, b in timing["quant"]) / steps
        res["forward_ms" + tag] = t_fwd
        res["backward_ms" + tag] = t_bwd
        res["forward_TFLOP/s" + tag] = fl_f / (t_fwd * 1e-3) / 1e12
        res["backward_TFLOP/s" + tag] = fl_b / (t_bwd * 1e-3) / 1e12
    res["timing"] = f"CUDA events over {steps} steps after {warmup} warm-up steps"
    del layers, flat
    torch.cuda.empty_cache()
    v, threads, desc, secs = oracle_sample(seconds_budget=8.0, rows=1024, toks=512, wl=wl)
    res["cpu_oracle"] = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc,
                         "seconds": secs}
    return res


def sub_tiny(device, peaks, reps=64):
    """The tiny layer (W 256x256 float32, 16 tokens, r = 8, alpha = 16): quantise +
    forward + backward per call, as CUDA-graph replays (the work is a few MFLOP,
    so the figure is a latency; launch-bound), next to the oracle on the same
    inputs."""
    import time as _time

    import torch

    import oracle as O
    from bit_nf4_quantized_27_b200 import binding as bd
    from bit_nf4_quantized_27_b200 import inputs as I

    wl = I.TINY
    w, x, a, b, dy = I.weight(wl), I.activations(wl), I.lora_a(wl), I.lora_b(wl), I.grad_output(wl)
    n, k = w.shape
    m, r = x.shape[0], a.shape[0]
    wc, xc, ac, bc, dyc = (t.to(device) for t in (w, x, a, b, dy))
    q = bd.NF4Weight(n, k, device)
    wsq = bd.new_workspace(bd.STATUS_BYTES, device)
    wsf = bd.new_workspace(bd.workspace_bytes(m, n, k, r, False), device)
    wsb = bd.new_workspace(bd.workspace_bytes(m, n, k, r, True), device)
    y = torch.empty(m, n, dtype=torch.bfloat16, device=device)
    t = torch.empty(2, m, r, dtype=torch.bfloat16, device=device)
    dx = torch.empty(m, k, dtype=torch.bfloat16, device=device)
    da = torch.empty(r, k, dtype=torch.float32, device=device)
    db = torch.empty(n, r, dtype=torch.float32, device=device)

    def calls():
        for _ in range(reps):
            bd.quantize(wc, out=q, ws=wsq)
            bd.linear_fwd(q, ac, bc, wl.alpha, xc, ws=wsf, out=y, t_out=t)
            bd.linear_bwd(q, ac, bc, wl.alpha, xc, dyc, t, ws=wsb, outs=(dx, da, db), grad_dtype=torch.float32)

    us = graph_time_us(calls) / reps
    fl = sum(layer_flops(m, n, k, r))
    wf, xf, af, bf, dyf = (t_.float().numpy() for t_ in (w, x, a, b, dy))
    times = []
    for _ in range(20):
        t0 = _time.perf_counter()
        qo = O.quantize(wf, n, k)
        wd = O.dequantize(qo["codes"], qo["scale_codes"], qo["c2"], n, k)
        _, to = O.linear_fwd(wd, af, bf, xf, wl.alpha, r)
        O.linear_bwd(wd, af, bf, xf, dyf, wl.alpha, r, to)
        times.append(time.perf_counter() - t0)
    cpu_us = statistics.median(times) * 1e6
    return {"us_per_call": us, "TFLOP/s": fl / (us * 1e-6) / 1e12, "flops_per_call": fl,
            "bound": "launch latency (one quantise, one forward and the backward kernels per call)",
            "timing": f"CUDA graph of {reps} calls (quantise + forward + backward)",
            "cpu_oracle": {"us_per_call": cpu_us, "kind": "oracle", "sample": "the whole call, median of 20"}}


def sub_quant(device, peaks):
    """Quantise / dequantise sweep (4096x4096 and 11008x4096 bf16): GB/s, timed as
    CUDA-graph replays over weight copies larger than L2 in total."""
    import torch

    from bit_nf4_quantized_27_b200 import binding as bd

    res = {}
    for n, k in ((4096, 4096), (11008, 4096)):
        copies = 4 if n > 4096 else 10  # 453 MB / 420 MB touched per rotation, over 3x L2
        ws_ = [(torch.randn(n, k, device=device) * 0.02).to(torch.bfloat16) for _ in range(copies)]
        qs = [bd.NF4Weight(n, k, device) for _ in range(copies)]
        outs = [torch.empty(n, k, dtype=torch.bfloat16, device=device) for _ in range(copies)]
        st = bd.new_workspace(256, device)
        reps = 4 * copies
        nbytes = n * k * 2 + n * k // 2 + n * k // 64 + 4 * ((n * k // 64 + 255) // 256)
        for name, fn in (("quantize", lambda i: bd.quantize(ws_[i % copies], out=qs[i % copies], ws=st)),
                         ("dequantize", lambda i: bd.dequantize(qs[i % copies], out=outs[i % copies]))):
            for i in range(copies):
                fn(i)
            torch.cuda.synchronize()
            us = graph_time_us(lambda: [fn(i) for i in range(reps)]) / reps
            gbs = nbytes / (us * 1e-6) / 1e9
            res[f"{name}_{n}x{k}"] = {"us": us, "GB/s": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"]}
        del ws_, qs, outs
    return res


def sub_adapters(device, peaks):
    """The steps after backward: merged export of an 8192x8192 NF4 weight with
    an r = 64 adapter (CUDA graph over 4 weight copies), and one AdamW step over
    the 65B-shaped block's adapters (flat fp32 with the bf16 copy).  GB/s of
    algorithmic bytes against the measured HBM copy bandwidth."""
    import torch

    from bit_nf4_quantized_27_b200 import binding as bd

    res = {}
    n = k = 8192
    r = 64
    copies = 4
    qs = []
    for _ in range(copies):
        w = (torch.randn(n, k, device=device) * 0.02).to(torch.bfloat16)
        qs.append(bd.quantize(w))
        del w
    a = (torch.randn(r, k, device=device) / k ** 0.5).to(torch.bfloat16)
    b = (torch.randn(n, r, device=device) * 0.01).to(torch.bfloat16)
    outs = [torch.empty(n, k, dtype=torch.bfloat16, device=device) for _ in range(copies)]
    for i in range(copies):
        bd.merge(qs[i], a, b, 16.0, out=outs[i])
    torch.cuda.synchronize()
    reps = 2 * copies
    us = graph_time_us(lambda: [bd.merge(qs[i % copies], a, b, 16.0, out=outs[i % copies]) for i in range(reps)]) / reps
    nbytes = n * k * 2 + n * k // 2 + n * k // 64 + 4 * (n * k // 64 // 256) + 2 * r * (n + k)
    res["merge_8192x8192_r64"] = {"us": us, "GB/s": nbytes / (us * 1e-6) / 1e9,
                                  "frac_of_hbm": nbytes / (us * 1e-6) / 1e9 / peaks["hbm_gbs"],
                                  "tensor_TFLOP/s": 2 * n * k * r / (us * 1e-6) / 1e12}
    del qs, outs
    torch.cuda.empty_cache()
    npar = sum(r * kk + nn * r for nn, kk in ((8192, 8192),) * 4 + ((22016, 8192),) * 2 + ((8192, 22016),))
    p, g, m, v = (torch.randn(npar, device=device) * 0.01 for _ in range(4))
    v.abs_()
    p16 = torch.empty(npar, dtype=torch.bfloat16, device=device)
    for i in range(3):
        bd.adamw_step(p, g, m, v, i + 1, 1e-4, weight_decay=0.01, p_bf16=p16)
    torch.cuda.synchronize()
    st, en = cuda_timer()
    steps = 20
    st.record()
    for i in range(steps):
        bd.adamw_step(p, g, m, v, i + 4, 1e-4, weight_decay=0.01, p_bf16=p16)
    en.record()
    torch.cuda.synchronize()
    us = st.elapsed_time(en) * 1e3 / steps
    nbytes = npar * (16 + 12 + 2)
    res["adamw_65b_block_adapters"] = {"params": npar, "us": us, "GB/s": nbytes / (us * 1e-6) / 1e9,
                                       "frac_of_hbm": nbytes / (us * 1e-6) / 1e9 / peaks["hbm_gbs"]}
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-sub", action="store_true", help="skip the GEMV / quantise / 7B-block side measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--ref-seconds", type=float, default=20.0)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank)
        return

    import torch

    from bit_nf4_quantized_27_b200 import binding as bd
    from bit_nf4_quantized_27_b200 import inputs as I

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    bd.lib()
    peaks, peaks_kind = load_peaks()
    wl = I.L65B_BLOCK
    layers, flat = build_block(wl, device, rank)
    fl_f = sum(layer_flops(wl.m, d["n"], d["k"], wl.r)[0] for d in layers)
    fl_b = sum(layer_flops(wl.m, d["n"], d["k"], wl.r)[1] for d in layers)

    def barrier():
        if world > 1:
            import torch.distributed as dist

            dist.barrier()

    for _ in range(args.warmup):
        run_step(layers, wl, flat, world)
    torch.cuda.synchronize()
    for d in layers:
        st = bd.read_status(d["ws_f"]) or bd.read_status(d["ws_b"])
        if st:
            raise RuntimeError(f"device status {bd.STATUS_NAMES[st]} on layer {d['name']}")

    # ---------------- timed region (device-resident inputs)
    timing = {"quant": [], "fwd": [], "bwd": []}
    sampler = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    s, e = cuda_timer()
    s.record()
    for _ in range(args.steps):
        run_step(layers, wl, flat, world, timing)
    e.record()
    # the training step proper: the weights stay quantised from the steps above
    s_nq, e_nq = cuda_timer()
    s_nq.record()
    for _ in range(args.steps):
        run_step(layers, wl, flat, world, quant=False)
    e_nq.record()
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    ms = s.elapsed_time(e) / args.steps
    ms_nq = s_nq.elapsed_time(e_nq) / args.steps
    if world > 1:
        import torch.distributed as dist

        t = torch.tensor([ms, ms_nq], device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms, ms_nq = (float(v) for v in t.tolist())
    value = world * (fl_f + fl_b) / (ms * 1e-3) / 1e12
    value_nq = world * (fl_f + fl_b) / (ms_nq * 1e-3) / 1e12
    t_fwd = sum(a.elapsed_time(b) for a, b in timing["fwd"]) / args.steps
    t_bwd = sum(a.elapsed_time(b) for a, b in timing["bwd"]) / args.steps
    t_q = sum(a.elapsed_time(b) for a, b in timing["quant"]) / args.steps

    # ---------------- end to end: inputs from pinned host memory, grads back
    host_x = [d["x"].cpu().pin_memory() for d in layers]
    host_dy = [d["dy"].cpu().pin_memory() for d in layers]
    host_g = torch.empty(flat.numel(), dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * 2 for t in host_x + host_dy)
    d2h = host_g.numel() * 4

    # Each step copies its inputs on a copy stream, in the order the step consumes
    # them (X of every layer, then dY from the last layer down), and each layer
    # waits only for its own tensors, so the copies overlap the compute.  The
    # copy stream first waits for the previous step to finish with the buffers.
    copy_stream = torch.cuda.Stream(device=device)

    def e2e_step():
        cur = torch.cuda.current_stream()
        copy_stream.wait_stream(cur)
        ev_x, ev_dy = [], [None] * len(layers)
        with torch.cuda.stream(copy_stream):
            for d, hx in zip(layers, host_x):
                d["x"].copy_(hx, non_blocking=True)
                ev_x.append(torch.cuda.Event())
                ev_x[-1].record(copy_stream)
            for i in reversed(range(len(layers))):
                layers[i]["dy"].copy_(host_dy[i], non_blocking=True)
                ev_dy[i] = torch.cuda.Event()
                ev_dy[i].record(copy_stream)
        run_step(layers, wl, flat, world, ready=(ev_x, ev_dy))
        host_g.copy_(flat, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    s2, e2 = cuda_timer()
    s2.record()
    e2e_steps = max(3, args.steps // 2)
    for _ in range(e2e_steps):
        e2e_step()
    e2.record()
    torch.cuda.synchronize()
    ms_e2e = s2.elapsed_time(e2) / e2e_steps
    if world > 1:
        import torch.distributed as dist

        t = torch.tensor([ms_e2e], device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_e2e = float(t.item())
    e2e_value = world * (fl_f + fl_b) / (ms_e2e * 1e-3) / 1e12

    fwd_tf = fl_f / (t_fwd * 1e-3) / 1e12
    bwd_tf = fl_b / (t_bwd * 1e-3) / 1e12
    # The timed region is about 0.1 s with SM clocks at their maximum (see
    # `clocks`), the conditions of the burst measurement; the sustained figure
    # (a seconds-long loop that settled near 1.3 GHz) is reported beside it.
    peak_tc = peaks["bf16_tflops"]
    peak_sus = peaks["bf16_tflops_sustained"]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_config(),
        "roofline": {"bound": "tensor", "kernel": "NF4 fused tensor-core GEMM on CTA pairs, forward call (T = X A^T "
                                                  "with split K, then the fused dequant GEMM with the LoRA K steps), "
                                                  "all 7 layers",
                     "achieved": fwd_tf, "peak": peak_tc, "unit": "TFLOP/s", "frac": fwd_tf / peak_tc,
                     "traffic": fused_fwd_traffic(), "traffic_unit": "bytes per fused forward launch",
                     "peak_kind": f"{peaks_kind} bf16 dense, burst",
                     "frac_of_sustained": fwd_tf / peak_sus, "step_frac": value / world / peak_tc},
        "breakdown_ms_per_step": {"quantize": t_q, "forward": t_fwd, "backward": t_bwd,
                                  "forward_TFLOP/s": fwd_tf, "backward_TFLOP/s": bwd_tf},
        "train_step_no_quant": {"ms_per_step": ms_nq, "TFLOP/s": value_nq,
                                "frac_of_bf16": value_nq / world / peak_tc,
                                "note": "weights quantised once at load (QLoRA), forward + backward of the 7 layers"},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": ms_e2e,
                "copies": "per layer from pinned memory on a copy stream, overlapping the step's compute; "
                          "gradients read back after the step"},
        "gpu_launches": launches_per_step(len(layers)) * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and not args.no_sub:
        del host_x, host_dy
        layers.clear()
        torch.cuda.empty_cache()
        line["sub"] = {"gemv_11008x4096_r64": sub_gemv(device, peaks), "quant_sweep": sub_quant(device, peaks),
                       "adapter_steps": sub_adapters(device, peaks),
                       "block_7b_m2048_r64": sub_block7b(device, peaks),
                       "tiny_256x256_m16_r8": sub_tiny(device, peaks)}
    if rank == 0 and world == 1 and not args.no_cpu:
        v, threads, desc, secs = oracle_sample()
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc,
                                "seconds": secs}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
