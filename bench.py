#!/usr/bin/env python3
"""Benchmark of the QLoRA NF4 + double-quant frozen-base linear layer on B200.

One step = one pass of the whole hot path over one batch of synthetic input,
for each of the three LLaMA-7B-shaped linears (h, o) = (4096, 4096),
(4096, 11008), (11008, 4096) at M = 4096 tokens, r = 64, s = 16/64:
  quantize to NF4 + double-quantize the constants -> dequantize to bf16 ->
  fused forward Y = X W' + s X L1 L2 -> backward dX, dL1, dL2 ->
  small-M (M = 16) forward on the same weight.
With N > 1 ranks each rank runs its own batch (weak scaling) and the LoRA
gradients are summed over ranks with one NCCL all-reduce per layer.

Prints one JSON line (rank 0).  `value` is the fwd+bwd TFLOP/s of the whole
job (4 M h o + 6 M r (h + o) per layer per rank) divided by the device time of
the whole step, max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "QLoRA linear fwd+bwd TFLOP/s & % bf16 peak; NF4 quant/dequant GB/s & % HBM"
WORKLOAD = {
    "workload": "llama7b_shaped_linears_fwd_bwd",
    "M": 4096,
    "layers": [[4096, 4096], [4096, 11008], [11008, 4096]],
    "r": 64,
    "s": 0.25,
    "small_m": 16,
}
# Bulk quantize / dequant workload: the 7 linear weights of one LLaMA-65B-shaped
# decoder layer (d = 8192, ffn = 22016; (h, o) per weight, stored W^T [o][h]),
# N(0, 0.02) with 0.1 % of entries set to +-8 sigma.
BULK = {
    "workload": "llama65b_layer_bulk_quantize_dequant",
    "weights": [[8192, 8192]] * 4 + [[8192, 22016]] * 2 + [[22016, 8192]],
    "outlier_frac": 0.001,
}
# Small-M (decode) forward workload: 65B-shaped weights, M in {1, 4, 16}, r = 64.
DECODE = {"workload": "llama65b_decode_forward", "weights": [[8192, 8192], [8192, 22016]], "M": [1, 2, 4, 16],
          "r": 64, "s": 0.25}
# All-linear LoRA stack of one LLaMA-13B-shaped decoder layer (d = 5120,
# ffn = 13824): q, k, v, o, gate, up, down in sequence, M = 8192, r = 64, fwd + bwd.
STACK = {"workload": "llama13b_layer_stack_fwd_bwd", "M": 8192,
         "layers": [[5120, 5120]] * 4 + [[5120, 13824]] * 2 + [[13824, 5120]], "r": 64, "s": 0.25}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DQ_BYTES_PER_PARAM = 0.5 + 1 / 64 + 4 / (64 * 256)  # packed codes + FP8 constants + fp32 group scales


def fwd_bwd_flops(M, h, o, r):
    return 4 * M * h * o + 6 * M * r * (h + o)


def fused_fwd_flops(M, h, o, r):
    return 2 * M * h * o + 2 * M * r * o


def fused_bwd_flops(M, h, o, r):
    return 2 * M * h * o + 2 * M * r * h


def small_m_bytes(M, h, o, r):
    return DQ_BYTES_PER_PARAM * h * o + 2 * r * (h + o) + 2 * M * (h + o)


def kernel_source_hash():
    """sha256 (16 hex digits) of the code that defines the headline's GEMM
    kernel (pairgemm.cuh, the pair-tile bf16 GEMM) plus common.cuh, with
    comments and blank lines left out.  Ties stored ncu counters to a kernel
    version."""
    import hashlib
    import re
    csrc = os.path.join(ROOT, "bit_nf4_quantized_blockwise_b200", "csrc")
    h = hashlib.sha256()
    for name in ("pairgemm.cuh", "common.cuh"):
        with open(os.path.join(csrc, name)) as f:
            for line in f:
                code = re.sub(r"//.*$", "", line).strip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


TRAFFIC_PROFILE = os.path.join("profiles", "pair_gemm_traffic_llama7b.txt")


def stored_traffic():
    """DRAM bytes per GEMM launch from the committed ncu summary, or None when
    the summary is missing or was taken on a different kernel version."""
    path = os.path.join(ROOT, TRAFFIC_PROFILE)
    try:
        fields = {}
        with open(path) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    fields[k.strip()] = v.strip()
        if fields.get("kernel_source_sha256_16") != kernel_source_hash():
            return None
        return float(fields["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def tensor_peak(peaks, timed_s, clocks):
    """The dense bf16 peak a tensor-bound number is compared with: the burst
    figure (a GEMM timed alone, unthrottled) when the timed region is short and
    the clock record saw no power capping, else the sustained figure (a long
    back-to-back loop under the power cap).  Returns (peak, which)."""
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    capped = "sw_power_cap" in (clocks or {}).get("reasons", [])
    if timed_s < 1.0 and not capped:
        return burst, "bf16_tflops (burst: timed region %.3f s, no sw_power_cap)" % timed_s
    return sustained, "bf16_tflops_sustained (timed region %.3f s%s)" % (timed_s, ", sw_power_cap" if capped else "")


# ---------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.file = None
        self.target = None
        try:
            props = torch.cuda.get_device_properties(device_index)
            uuid = str(getattr(props, "uuid", ""))
            if uuid:
                self.target = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.target = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            cmd = ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits", "-lms", "50"]
            if self.target:
                cmd += ["-i", self.target]
            self.proc = subprocess.Popen(cmd, stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.file.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        os.unlink(self.file.name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "power_w_max": max(power),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------- our arm

class LayerState:
    """Device buffers of one linear layer (all allocated before timing)."""

    def __init__(self, q, M, h, o, r, s, small_m, seed, dev, codebook):
        import synth
        from bit_nf4_quantized_blockwise_b200 import dp
        self.h, self.o, self.r, self.s, self.M, self.small_m = h, o, r, s, M, small_m
        self.W_t_host = synth.weight_t(o, h, seed=seed, tag=f"W{h}x{o}").pin_memory()
        self.X_host = synth.activations(M, h, seed=seed, tag=f"X{h}").pin_memory()
        self.dY_host = synth.activations(M, o, seed=seed, tag=f"dY{o}").pin_memory()
        L1, L2 = synth.lora_factors(h, r, o, seed=seed)
        self.L1_host, self.L2_host = L1.pin_memory(), L2.pin_memory()
        self.W_t = self.W_t_host.to(dev)
        self.X = self.X_host.to(dev)
        self.dY = self.dY_host.to(dev)
        self.L1 = self.L1_host.to(dev)
        self.L2 = self.L2_host.to(dev)
        self.Xs = self.X[:small_m].contiguous()
        n = o * h
        self.codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
        self.absmax = torch.empty(n // 64, dtype=torch.float32, device=dev)
        self.fp8 = torch.empty(n // 64, dtype=torch.uint8, device=dev)
        self.sc = torch.empty(n // 64 // 256, dtype=torch.float32, device=dev)
        self.mu = torch.empty(1, dtype=torch.float32, device=dev)
        self.dq_ws = torch.empty(256, dtype=torch.uint8, device=dev)
        self.Wq = q.NF4Weight(self.codes, self.fp8, self.sc, self.mu, o, h, tuple(float(v) for v in codebook))
        self.Wd = torch.empty(o, h, dtype=torch.bfloat16, device=dev)
        self.Y = torch.empty(M, o, dtype=torch.float32, device=dev)
        self.T = torch.empty(M, r, dtype=torch.float32, device=dev)
        self.dX = torch.empty(M, h, dtype=torch.float32, device=dev)
        self.grads, self.dL1, self.dL2 = dp.lora_grad_buffers(h, o, r, dev)
        self.Ys = torch.empty(small_m, o, dtype=torch.float32, device=dev)
        L = q.lib()
        wsb = max(L.qlora_linear_fwd_workspace_size(o, h, M, r), L.qlora_linear_bwd_workspace_size(o, h, M, r))
        self.ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
        # host buffers of the step's results, for the end-to-end pass
        self.Y_out = torch.empty_like(self.Y, device="cpu").pin_memory()
        self.dX_out = torch.empty_like(self.dX, device="cpu").pin_memory()
        self.grads_out = torch.empty_like(self.grads, device="cpu").pin_memory()
        self.Ys_out = torch.empty_like(self.Ys, device="cpu").pin_memory()

    def h2d_bytes(self):
        return sum(t.numel() * t.element_size() for t in (self.W_t_host, self.X_host, self.dY_host,
                                                          self.L1_host, self.L2_host))

    def d2h_bytes(self):
        return sum(t.numel() * t.element_size() for t in (self.Y_out, self.dX_out, self.grads_out, self.Ys_out))

    def upload(self):
        self.W_t.copy_(self.W_t_host, non_blocking=True)
        self.X.copy_(self.X_host, non_blocking=True)
        self.dY.copy_(self.dY_host, non_blocking=True)
        self.L1.copy_(self.L1_host, non_blocking=True)
        self.L2.copy_(self.L2_host, non_blocking=True)
        self.Xs.copy_(self.X[: self.small_m])

    def download(self):
        self.Y_out.copy_(self.Y, non_blocking=True)
        self.dX_out.copy_(self.dX, non_blocking=True)
        self.grads_out.copy_(self.grads, non_blocking=True)
        self.Ys_out.copy_(self.Ys, non_blocking=True)


def run_step(q, layers, codebook, dp, group):
    for L in layers:
        q.qlora_quantize_nf4(L.W_t, codebook, codes=L.codes, absmax=L.absmax)
        q.qlora_double_quant(L.absmax, absmax_fp8=L.fp8, dq_scale=L.sc, dq_mean=L.mu, ws=L.dq_ws)
        q.qlora_dequant(L.Wq, out=L.Wd)
        q.qlora_linear_fwd(L.Wq, L.X, L.L1, L.L2, L.s, Y=L.Y, T_save=L.T, ws=L.ws)
        q.qlora_linear_bwd(L.Wq, L.X, L.dY, L.L1, L.L2, L.s, T_saved=L.T, dX=L.dX, dL1=L.dL1, dL2=L.dL2,
                           ws=L.ws)
        q.qlora_linear_fwd(L.Wq, L.Xs, L.L1, L.L2, L.s, Y=L.Ys, save_T=False, ws=L.ws)
        dp.allreduce_lora_grads(L.grads, group)


def time_steps(fn, steps, dev):
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    start.record()
    for _ in range(steps):
        fn()
    stop.record()
    torch.cuda.synchronize(dev)
    return start.elapsed_time(stop)


def graph_time(fn, n, dev):
    """Device time (ms) of one fn() call: n calls captured in a CUDA graph and
    replayed, so that host-side launch cost does not pad short calls.  Falls
    back to timing the calls eagerly if the capture fails."""
    try:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize(dev)
        with torch.cuda.graph(g):
            for _ in range(n):
                fn()
        g.replay()
        torch.cuda.synchronize(dev)
        ms = time_steps(g.replay, 3, dev) / 3
        del g
        return ms / n, f"CUDA graph of {n} calls, replayed 3 times"
    except Exception as e:  # noqa: BLE001
        torch.cuda.synchronize(dev)
        return time_steps(fn, n, dev) / n, f"eager ({type(e).__name__}: graph capture failed)"


def max_over_ranks(x, dev, world):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measure_bulk(q, dev, codebook, hbm_peak, reps=5):
    """Quantize + double-quantize, then dequantize, the 7 weights of the bulk
    workload; CUDA events over `reps` passes of all 7 (inputs 1.6 GB > L2)."""
    import synth
    states = []
    for i, (h, o) in enumerate(BULK["weights"]):
        W = synth.weight_t(o, h, seed=100 + i, tag=f"Wb{h}x{o}", outlier_frac=BULK["outlier_frac"]).to(dev)
        n = o * h
        codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
        absmax = torch.empty(n // 64, dtype=torch.float32, device=dev)
        fp8 = torch.empty(n // 64, dtype=torch.uint8, device=dev)
        sc = torch.empty(n // 64 // 256, dtype=torch.float32, device=dev)
        mu = torch.empty(1, dtype=torch.float32, device=dev)
        ws = torch.empty(256, dtype=torch.uint8, device=dev)
        Wq = q.NF4Weight(codes, fp8, sc, mu, o, h, tuple(float(v) for v in codebook))
        states.append((W, codes, absmax, fp8, sc, mu, ws, Wq, torch.empty_like(W)))

    def quant_all():
        for W, codes, absmax, fp8, sc, mu, ws, Wq, out in states:
            q.qlora_quantize_nf4(W, codebook, codes=codes, absmax=absmax)
            q.qlora_double_quant(absmax, absmax_fp8=fp8, dq_scale=sc, dq_mean=mu, ws=ws)

    def dequant_all():
        for W, codes, absmax, fp8, sc, mu, ws, Wq, out in states:
            q.qlora_dequant(Wq, out=out)

    quant_all()
    dequant_all()
    torch.cuda.synchronize(dev)
    q.qlora_check_status(dev)
    tq = time_steps(quant_all, reps, dev) / reps
    td = time_steps(dequant_all, reps, dev) / reps
    q.qlora_trace_enable(True)
    quant_all()
    dequant_all()
    torch.cuda.synchronize(dev)
    tr = q.qlora_trace_read()
    q.qlora_trace_enable(False)
    params = sum(h * o for h, o in BULK["weights"])
    b = params * (2 + DQ_BYTES_PER_PARAM)
    del states
    torch.cuda.empty_cache()
    return {
        "params": params, "bytes_each_way": b,
        "quantize_dq": {"gbs": round(b / (tq * 1e-3) / 1e9, 1), "frac_hbm": round(b / (tq * 1e-3) / 1e9 / hbm_peak, 4),
                        "ms": round(tq, 4)},
        "dequant": {"gbs": round(b / (td * 1e-3) / 1e9, 1), "frac_hbm": round(b / (td * 1e-3) / 1e9 / hbm_peak, 4),
                    "ms": round(td, 4)},
        "kernel_ms": {k: round(v[0], 4) for k, v in tr.items() if v[1]},
        "kernel_launches": {k: int(v[1]) for k, v in tr.items() if v[1]},
        "l2": "inputs 1.6 GB, larger than L2",
    }


def measure_stack(q, dev, codebook, peaks, reps=5, dropout=0.0):
    """Forward + backward of the 7 linears of the 13B-shaped layer in sequence
    (weights quantized once beforehand; synthetic activations per linear),
    optionally with LoRA dropout of rate `dropout` on every adapter input."""
    M, r, s = STACK["M"], STACK["r"], STACK["s"]
    layers = [LayerState(q, M, h, o, r, s, 1, 5000 + i, dev, codebook) for i, (h, o) in enumerate(STACK["layers"])]
    for L in layers:
        q.qlora_quantize_nf4(L.W_t, codebook, codes=L.codes, absmax=L.absmax)
        q.qlora_double_quant(L.absmax, absmax_fp8=L.fp8, dq_scale=L.sc, dq_mean=L.mu, ws=L.dq_ws)

    if dropout:
        Lb = q.lib()
        for L in layers:
            wsb = Lb.qlora_linear_bwd_dropout_workspace_size(L.o, L.h, M, r)
            if L.ws.numel() < wsb:
                L.ws = torch.empty(wsb, dtype=torch.uint8, device=dev)

    def step():
        for i, L in enumerate(layers):
            q.qlora_linear_fwd(L.Wq, L.X, L.L1, L.L2, L.s, Y=L.Y, T_save=L.T, ws=L.ws, dropout=dropout, seed=11 + i)
            q.qlora_linear_bwd(L.Wq, L.X, L.dY, L.L1, L.L2, L.s, T_saved=L.T, dX=L.dX, dL1=L.dL1, dL2=L.dL2,
                               ws=L.ws, dropout=dropout, seed=11 + i)
    for _ in range(3):
        step()
    torch.cuda.synchronize(dev)
    q.qlora_check_status(dev)
    sampler = ClockSampler(dev.index)
    sampler.start()
    total = time_steps(step, reps, dev)
    clocks = sampler.stop()
    ms = total / reps
    flops = sum(fwd_bwd_flops(M, h, o, r) for h, o in STACK["layers"])
    tf = flops / (ms * 1e-3) / 1e12
    peak, which = tensor_peak(peaks, total * 1e-3, clocks)
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    del layers
    torch.cuda.empty_cache()
    return {"ms_per_step": round(ms, 4), "tflops": round(tf, 1), "frac_tensor": round(tf / peak, 4),
            "peak_used": which, "frac_of_burst": round(tf / burst, 4), "frac_of_sustained": round(tf / sustained, 4),
            "flops_per_step": int(flops), "clocks": clocks, "lora_dropout": dropout, "l2": "operands larger than L2"}


def measure_merge(q, dev, codebook, hbm_peak, reps=10):
    """Adapter merge W_m = bf16(W' + s L1 L2) on the three LLaMA-7B-shaped
    weights (r = 64): algorithmic bytes (packed weight 0.516 B/param + bf16
    output 2 B/param + the two factors) and the rank-r flops 2 r h o."""
    import synth
    r, s = WORKLOAD["r"], WORKLOAD["s"]
    states = []
    for i, (h, o) in enumerate(WORKLOAD["layers"]):
        W = synth.weight_t(o, h, seed=300 + i, tag=f"Wm{h}x{o}").to(dev)
        Wq = q.quantize_weight(W, codebook)
        L1, L2 = (t.to(dev) for t in synth.lora_factors(h, r, o, seed=300 + i))
        states.append((Wq, L1, L2, torch.empty(o, h, dtype=torch.bfloat16, device=dev)))

    def run():
        for Wq, L1, L2, out in states:
            q.qlora_merge_bf16(Wq, L1, L2, s, out=out)
    run()
    torch.cuda.synchronize(dev)
    q.qlora_check_status(dev)
    ms = time_steps(run, reps, dev) / reps
    params = sum(h * o for h, o in WORKLOAD["layers"])
    b = params * (DQ_BYTES_PER_PARAM + 2) + sum(2 * r * (h + o) for h, o in WORKLOAD["layers"])
    flops = sum(2 * r * h * o for h, o in WORKLOAD["layers"])
    del states
    torch.cuda.empty_cache()
    gbs = b / (ms * 1e-3) / 1e9
    return {"ms": round(ms, 4), "gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm_peak, 4),
            "tflops_rank_r": round(flops / (ms * 1e-3) / 1e12, 1), "bytes": int(b),
            "l2": "weights and outputs 3 x 67-180 MB per pass, larger than L2 together"}


def measure_optimizer(q, dev, hbm_peak, reps=10):
    """Paged AdamW step (global-norm clipping + update + bf16 copies) over the
    LoRA factors of the 13B-shaped layer stack (r = 64, 7 linears): state
    resident on the device, and state evicted to host RAM before every step
    (the worst case of a memory spike).  Algorithmic bytes per parameter:
    read p, g, m, v and write p, m, v (fp32) plus the bf16 copy, 30 B."""
    from bit_nf4_quantized_blockwise_b200.paged import AdamWConfig, PagedAdamW
    r = STACK["r"]
    n = sum(r * (h + o) for h, o in STACK["layers"])   # every L1 [h][r] and L2 [r][o], one flat buffer
    g0 = torch.Generator().manual_seed(5)
    param = (torch.randn(n, generator=g0) * 0.01).to(dev)
    grad = (torch.randn(n, generator=g0) * 0.01).to(dev)
    copy = torch.empty(n, dtype=torch.bfloat16, device=dev)
    opt = PagedAdamW(param, AdamWConfig(), copy=copy)
    for _ in range(3):
        opt.step(grad)
    torch.cuda.synchronize(dev)
    q.qlora_check_status(dev)
    ms = time_steps(lambda: opt.step(grad), reps, dev) / reps

    def evicted_step():
        opt.evict()
        opt.step(grad)
    ms_ev = time_steps(evicted_step, reps, dev) / reps
    opt.close()
    b = 30 * n
    return {"params": int(n), "ms_resident": round(ms, 4), "gbs_resident": round(b / (ms * 1e-3) / 1e9, 1),
            "frac_hbm_resident": round(b / (ms * 1e-3) / 1e9 / hbm_peak, 4),
            "ms_evicted_each_step": round(ms_ev, 4),
            "note": "evicted: state prefetched to host RAM before every step and brought back by the next step"}


def measure_decode(q, dev, codebook, hbm_peak, calls=30, shapes=None, tokens=None):
    """Small-M forward on the decode workload; each call takes the next of
    several copies of the quantized weight so the weight stream is cold in L2.
    shapes / tokens restrict the rows (profiling of one case)."""
    import synth
    L = q.lib()
    out = {}
    r, s = DECODE["r"], DECODE["s"]
    for h, o in shapes or DECODE["weights"]:
        W = synth.weight_t(o, h, seed=7, tag=f"Wd{h}x{o}").to(dev)
        Wq0 = q.quantize_weight(W, codebook)
        del W
        wbytes = DQ_BYTES_PER_PARAM * h * o
        nrot = int(300e6 // wbytes) + 2
        Wqs = [q.NF4Weight(Wq0.codes.clone(), Wq0.absmax_fp8.clone(), Wq0.dq_scale.clone(), Wq0.dq_mean.clone(), o, h,
                           Wq0.codebook) for _ in range(nrot)]
        L1, L2 = (t.to(dev) for t in synth.lora_factors(h, r, o, seed=7))
        for M in tokens or DECODE["M"]:
            X = synth.activations(M, h, seed=7, tag=f"Xd{h}").to(dev)
            Y = torch.empty(M, o, dtype=torch.float32, device=dev)
            ws = torch.empty(L.qlora_linear_fwd_workspace_size(o, h, M, r), dtype=torch.uint8, device=dev)
            it = [0]

            def call():
                q.qlora_linear_fwd(Wqs[it[0] % nrot], X, L1, L2, s, Y=Y, save_T=False, ws=ws)
                it[0] += 1
            for _ in range(3):
                call()
            torch.cuda.synchronize(dev)
            q.qlora_check_status(dev)
            t_call, how = graph_time(call, calls, dev)
            q.qlora_trace_enable(True)
            for _ in range(calls):
                call()
            torch.cuda.synchronize(dev)
            tr = q.qlora_trace_read()
            q.qlora_trace_enable(False)
            b = small_m_bytes(M, h, o, r)
            k_ms = tr["small_m_fwd"][0] / tr["small_m_fwd"][1]
            out[f"{h}x{o}_M{M}"] = {
                "small_m_kernel_us": round(k_ms * 1e3, 2), "small_m_gbs": round(b / (k_ms * 1e-3) / 1e9, 1),
                "small_m_frac_hbm": round(b / (k_ms * 1e-3) / 1e9 / hbm_peak, 4),
                "call_us": round(t_call * 1e3, 2), "call_gbs": round(b / (t_call * 1e-3) / 1e9, 1),
                "call_frac_hbm": round(b / (t_call * 1e-3) / 1e9 / hbm_peak, 4), "call_timing": how,
                "bytes": int(b)}
        del Wqs, Wq0
        torch.cuda.empty_cache()
    out["l2"] = "weight copies rotated per call, more than L2 in total"
    return out


def run_ours(args, rank, world, dev):
    import torch.distributed as dist

    import bit_nf4_quantized_blockwise_b200 as q
    from bit_nf4_quantized_blockwise_b200 import build as qbuild
    from bit_nf4_quantized_blockwise_b200 import dp

    if rank == 0:
        qbuild.build()
    if world > 1:
        dist.barrier()
    q.lib()
    codebook = q.qlora_nf4_codebook()
    if args.only == "stack":
        peaks, _ = load_peaks()
        return {"workload": STACK["workload"], "stack": measure_stack(q, dev, codebook, peaks, reps=args.steps)}
    if args.only in ("merge", "optim"):
        peaks, _ = load_peaks()
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        if args.only == "merge":
            return {"workload": "adapter_merge_llama7b", "merge": measure_merge(q, dev, codebook, hbm)}
        return {"workload": "paged_adamw_13b_stack", "optim": measure_optimizer(q, dev, hbm)}
    if args.only in ("bulk", "decode"):
        # profiling entry: one of the secondary workloads alone
        peaks, _ = load_peaks()
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        if args.only == "bulk":
            return {"workload": BULK["workload"], "bulk": measure_bulk(q, dev, codebook, hbm, reps=args.steps)}
        shapes = [[int(v) for v in args.decode_shape.split("x")]] if args.decode_shape else None
        tokens = [int(v) for v in args.decode_m.split(",")] if args.decode_m else None
        return {"workload": DECODE["workload"],
                "decode": measure_decode(q, dev, codebook, hbm, calls=args.steps, shapes=shapes, tokens=tokens)}
    W = dict(WORKLOAD)
    if args.layers is not None:
        W["layers"] = [WORKLOAD["layers"][int(i)] for i in args.layers.split(",")]
    M, r, s, sm = W["M"], W["r"], W["s"], W["small_m"]
    layers = [LayerState(q, M, h, o, r, s, sm, 1000 * rank + i, dev, codebook) for i, (h, o) in enumerate(W["layers"])]
    group = None
    step = lambda: run_step(q, layers, codebook, dp, group)  # noqa: E731

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    q.qlora_check_status(dev)
    if world > 1:
        dist.barrier()

    # (1) headline: K whole steps, no tracing
    sampler = ClockSampler(dev.index)
    sampler.start()
    n0 = q.qlora_launch_count()
    if world > 1:
        dist.barrier()
    t_ms = time_steps(step, args.steps, dev)
    if world > 1:
        dist.barrier()
    launches = q.qlora_launch_count() - n0
    clocks = sampler.stop()
    t_ms = max_over_ranks(t_ms, dev, world)

    flops_step = sum(fwd_bwd_flops(M, h, o, r) for h, o in W["layers"])
    value = flops_step * world * args.steps / (t_ms * 1e-3) / 1e12
    if args.quick:
        return {"metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_ms / args.steps, 4),
                "config": dict(W, quick=True), "gpu_launches": int(launches), "clocks": clocks}

    # (2) per-kernel device times: the same K steps with launch tracing on
    q.qlora_trace_enable(True)
    time_steps(step, args.steps, dev)
    trace = q.qlora_trace_read()
    q.qlora_trace_enable(False)

    # (3) end to end: pinned host inputs -> device -> step -> host results
    e2e_steps = max(1, min(args.steps, 5))

    def e2e_step():
        for L in layers:
            L.upload()
        step()
        for L in layers:
            L.download()
    e2e_step()
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(time_steps(e2e_step, e2e_steps, dev), dev, world)
    q.qlora_check_status(dev)

    e2e_value = flops_step * world * e2e_steps / (e2e_ms * 1e-3) / 1e12

    peaks, peak_src = load_peaks()
    tc_peak, tc_which = tensor_peak(peaks, t_ms * 1e-3, clocks)
    tc_burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    tc_sust = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    K = args.steps
    fused_ms = trace["nf4_gemm_fwd"][0] + trace["nf4_gemm_bwd_dx"][0]
    fused_n = trace["nf4_gemm_fwd"][1] + trace["nf4_gemm_bwd_dx"][1]
    fused_flops = K * sum(fused_fwd_flops(M, h, o, r) + fused_bwd_flops(M, h, o, r) for h, o in W["layers"])
    achieved = fused_flops / (fused_ms * 1e-3) / 1e12 if fused_ms > 0 else None
    # the same products with the per-call dequantization of W' counted in
    wprime_ms = trace["nf4_dequant_wprime"][0]
    op_tflops = fused_flops / ((fused_ms + wprime_ms) * 1e-3) / 1e12 if fused_ms > 0 else None

    params = sum(h * o for h, o in W["layers"])
    q_ms = trace["nf4_quantize"][0] + trace["double_quant"][0]
    dq_ms = trace["nf4_dequant"][0]
    quant_bytes = K * params * (2 + DQ_BYTES_PER_PARAM)
    deq_bytes = K * params * (DQ_BYTES_PER_PARAM + 2)
    step_ms = t_ms / K
    rows = {
        "quantize_dq": {"gbs": quant_bytes / (q_ms * 1e-3) / 1e9 if q_ms else None,
                        "frac_hbm": (quant_bytes / (q_ms * 1e-3) / 1e9) / hbm_peak if q_ms else None,
                        "ms_per_step": q_ms / K, "bytes_per_param": 2 + DQ_BYTES_PER_PARAM},
        "dequant": {"gbs": deq_bytes / (dq_ms * 1e-3) / 1e9 if dq_ms else None,
                    "frac_hbm": (deq_bytes / (dq_ms * 1e-3) / 1e9) / hbm_peak if dq_ms else None,
                    "ms_per_step": dq_ms / K, "bytes_per_param": DQ_BYTES_PER_PARAM + 2},
        "nf4_gemm_fwd_bwd": {"tflops": achieved, "frac_tensor": achieved / tc_peak if achieved else None,
                             "frac_of_burst": achieved / tc_burst if achieved else None,
                             "frac_of_sustained": achieved / tc_sust if achieved else None,
                             "ms_per_step": fused_ms / K, "launches_per_step": fused_n / K,
                             "with_wprime_dequant": {"tflops": op_tflops,
                                                     "frac_of_burst": op_tflops / tc_burst if op_tflops else None,
                                                     "ms_per_step": (fused_ms + wprime_ms) / K}},
        "kernel_ms_per_step": {k: v[0] / K for k, v in trace.items()},
        "kernel_launches_per_step": {k: v[1] / K for k, v in trace.items()},
    }
    sm_ms = trace["small_m_fwd"][0]
    if sm_ms > 0:
        smb = K * sum(small_m_bytes(sm, h, o, r) for h, o in W["layers"])
        rows["small_m_fwd"] = {"gbs": smb / (sm_ms * 1e-3) / 1e9, "frac_hbm": smb / (sm_ms * 1e-3) / 1e9 / hbm_peak,
                               "ms_per_step": sm_ms / K}

    out = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,0.02) weights, N(0,1) activations, N(0,0.01) LoRA factors)",
        "config": dict(W, parallelism=f"dp{world}", tokens_per_rank=M, inputs_exceed_l2=True, l2_flush=False,
                       gemm_out_dtype="fp32"),
        "roofline": {"bound": "tensor",
                     "kernel": "pair_gemm_kernel: X W' and dY W'^T with the LoRA stages (6 launches per step; "
                               "W' dequantized into the workspace by a separate kernel, see rows)",
                     "achieved": round(achieved, 2) if achieved else None, "peak": tc_peak, "unit": "TFLOP/s",
                     "frac": round(achieved / tc_peak, 4) if achieved else None, "traffic": stored_traffic(),
                     "traffic_note": "DRAM read+write bytes per GEMM launch (mean over the 6 launches of a step) "
                                     "from " + TRAFFIC_PROFILE + "; null if the kernel changed since that capture",
                     "peak_source": f"{peak_src} {tc_which}",
                     "frac_of_burst": round(achieved / tc_burst, 4) if achieved else None,
                     "frac_of_sustained": round(achieved / tc_sust, 4) if achieved else None},
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": sum(L.h2d_bytes() for L in layers),
                "d2h_bytes_per_step": sum(L.d2h_bytes() for L in layers), "steps": e2e_steps},
        "gpu_launches": int(launches),
        "clocks": clocks,
        "rows": rows,
    }
    # the secondary workloads of the metric (1 GPU, after the timed step)
    if rank == 0 and world == 1:
        out["rows"]["bulk_65b_layer"] = dict(measure_bulk(q, dev, codebook, hbm_peak), config=BULK)
        out["rows"]["decode_65b"] = dict(measure_decode(q, dev, codebook, hbm_peak), config=DECODE)
        out["rows"]["stack_13b_layer"] = dict(measure_stack(q, dev, codebook, peaks), config=STACK)
        out["rows"]["stack_13b_layer_dropout_0.1"] = measure_stack(q, dev, codebook, peaks, dropout=0.1)
        out["rows"]["stack_13b_layer_dropout_0.05"] = measure_stack(q, dev, codebook, peaks, dropout=0.05)
        out["rows"]["adapter_merge_llama7b"] = measure_merge(q, dev, codebook, hbm_peak)
        out["rows"]["paged_adamw_13b_stack"] = measure_optimizer(q, dev, hbm_peak)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_budget)
    return out


# ---------------------------------------------------------------------------- oracle on the host

def _cores():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample_step(tokens, seed=7, which=None):
    """fp64 oracle forward + backward on `tokens` rows of the three linears
    (or of layer `which` only).  Returns the algorithmic flops processed."""
    import synth
    from oracle import nf4
    W = WORKLOAD
    flops = 0
    for i, (h, o) in enumerate(W["layers"]):
        if which is not None and i != which:
            continue
        Wt = _ORACLE_CACHE.setdefault(("W", h, o), synth.weight_t(o, h, seed=seed, tag=f"W{h}x{o}").double().numpy())
        L1, L2 = _ORACLE_CACHE.setdefault(("L", h, o), tuple(t.double().numpy() for t in synth.lora_factors(h, W["r"], o, seed=seed)))
        X = synth.activations(tokens, h, seed=seed + i, tag="Xs").double().numpy()
        dY = synth.activations(tokens, o, seed=seed + i, tag="dYs").double().numpy()
        nf4.lora_forward(X, Wt, L1, L2, W["s"])
        nf4.lora_backward(X, dY, Wt, L1, L2, W["s"])
        flops += fwd_bwd_flops(tokens, h, o, W["r"])
    return flops


_ORACLE_CACHE = {}


def oracle_quant_sample(n_elems=1 << 20, seed=7):
    """Oracle quantize + double-quant + dequant of n_elems weights; returns bytes moved (algorithmic)."""
    import synth
    from oracle import nf4
    cb = nf4.nf4_codebook()
    w = synth.weight_t(n_elems // 4096, 4096, seed=seed, tag="Wq", outlier_frac=0.001)
    bits = w.view(torch.uint16).numpy().reshape(-1)
    codes, absmax = nf4.quantize_blockwise(bits, cb)
    e, sc, mu = nf4.double_quant(absmax)
    nf4.dequant(nf4.pack_codes(codes), e, sc, mu, cb)
    return n_elems * (2 + DQ_BYTES_PER_PARAM) * 2


def cpu_baseline(budget_s=20.0):
    """The oracle, as it stands, on the host cores, on a bounded sample."""
    tokens = 256
    oracle_sample_step(8)  # warm the weight cache outside the timing
    t0 = time.perf_counter()
    flops = 0
    reps = 0
    while True:
        flops += oracle_sample_step(tokens)
        reps += 1
        if time.perf_counter() - t0 > budget_s * 0.7 or reps >= 8:
            break
    t_mm = time.perf_counter() - t0
    t1 = time.perf_counter()
    qbytes = oracle_quant_sample()
    t_q = time.perf_counter() - t1
    return {"value": round(flops / t_mm / 1e12, 6), "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
            "sample": f"fp64 oracle fwd+bwd of the 3 linears on {tokens} of {WORKLOAD['M']} tokens, {reps} reps "
                      f"({t_mm:.1f} s); weights bf16 widened to fp64",
            "quant_dequant_gbs": round(qbytes / t_q / 1e9, 4),
            "quant_sample": f"oracle quantize+DQ+dequant of 2^20 weights ({t_q:.1f} s)"}


def run_reference(args, rank, world):
    """The oracle as the reference arm: same metric, each step a bounded sample."""
    if rank != 0:
        return None
    tokens = 16
    oracle_sample_step(2)
    for i in range(args.warmup):
        oracle_sample_step(tokens, which=i % 3)
    t0 = time.perf_counter()
    flops = 0
    for i in range(args.steps):
        flops += oracle_sample_step(tokens, which=i % 3)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 6),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": dict(WORKLOAD, parallelism="host", tokens_per_step_sample=tokens),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
                         "sample": f"fp64 oracle fwd+bwd on {tokens} tokens of one of the 3 linears per step (rotating)"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--layers", type=str, default=None,
                    help="comma-separated layer indices to run (profiling cases); default all three")
    ap.add_argument("--only", choices=["bulk", "decode", "stack", "merge", "optim"], default=None,
                    help="profiling entry: run only the bulk quantize/dequant, the decode or the 13B layer-stack "
                         "workload")
    ap.add_argument("--decode-shape", type=str, default=None,
                    help="with --only decode: one weight shape HxO (e.g. 8192x22016) instead of all")
    ap.add_argument("--decode-m", type=str, default=None,
                    help="with --only decode: comma-separated token counts instead of all")
    ap.add_argument("--quick", action="store_true",
                    help="headline timing only: no traced pass, no end-to-end pass, no CPU baseline")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)

    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    try:
        out = run_ours(args, rank, world, dev)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
