#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 + DQ linear layer on B200.

Workload (one "step"): the seven linears of a LLaMA-7B layer (q, k, v, o:
4096x4096; gate, up: 4096->11008; down: 11008->4096), LoRA r=64, alpha=16
(s=0.25), 16x512 = 8192 tokens, synthetic seeded inputs:
  1. NF4 + Double-Quantization of the seven fp32 N(0, 0.02^2) weights,
  2. forward of the seven linears (Y = X W_hat^T + s X L1 L2),
  3. backward in reverse order (dX, dL1, dL2; no dW),
  4. with N > 1 ranks: all-reduce of the adapter gradients (data parallel).
Metric: algorithmic TFLOP/s of the linear forward+backward (4MKN + 6Mr(K+N)
per linear; quantization and dequantization work not counted), whole job.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from bit_nf4_quantized_02_b200.dp import FlatGrads  # noqa: E402
from synth import inputs, workloads  # noqa: E402

WL = workloads.LLAMA7B_LAYER
METRIC = "QLoRA NF4 linear fwd+bwd TFLOP/s"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def linear_flops(M, N, K, r):
    base = 2 * M * K * N
    lora = 2 * M * r * (K + N)
    return {"fwd": base + lora, "bwd": base + 2 * lora, "fwd_bwd": 2 * base + 3 * lora,
            "gemm_Y": base + 2 * M * r * N, "gemm_dX": base + 2 * M * r * K}


def step_flops(linears=None, M=WL.M, r=WL.r):
    return sum(linear_flops(M, l.n_out, l.k_in, r)["fwd_bwd"] for l in (linears or WL.linears))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "bit_nf4_quantized_02_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_indices):
        self.gpus = gpu_indices
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=5)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                idx = int(parts[0])
            except ValueError:
                continue
            if self.gpus and idx not in self.gpus:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- our arm
class Linear:
    def __init__(self, lin, X, dev, seed, wl=WL):
        M, r = wl.M, wl.r
        self.lin = lin
        N, K = lin.n_out, lin.k_in
        self.W = inputs.device_normal((N, K), inputs.WEIGHT_STD, seed, dev)
        self.L1 = inputs.device_normal((K, r), 1.0 / np.sqrt(K), seed + 1, dev, torch.bfloat16)
        self.L2 = inputs.device_normal((r, N), inputs.L2_STD, seed + 2, dev, torch.bfloat16)
        self.X = X
        self.dY = inputs.device_normal((M, N), 1.0, seed + 3, dev, torch.bfloat16)
        self.Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        self.T = torch.empty(M, 2 * r, dtype=torch.bfloat16, device=dev)
        self.dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
        self.q = None
        self.mask = None
        self.Xm = None         # masked adapter input, saved by the forward (LoRA dropout)


def device_dropout_mask(M, K, p, seed, dev):
    """Keep mask of LoRA dropout drawn on the device (seeded): int32 words
    [M, K/32], element 32 w + b kept in bit b of word w with probability 1 - p."""
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    keep = (torch.rand((M, K // 32, 32), generator=g, device=dev) >= p).to(torch.int64)
    words = (keep << torch.arange(32, device=dev, dtype=torch.int64)).sum(-1)
    return words.to(torch.uint32).view(torch.int32) if hasattr(torch, "uint32") else (
        torch.where(words >= 2 ** 31, words - 2 ** 32, words).to(torch.int32))


def build_layer(dev, rank, wl=WL):
    """The seven linears of one layer on independent seeded inputs."""
    M = wl.M
    hidden, mlp = wl.linears[0].k_in, wl.linears[4].n_out
    base = wl.seed + 1000 * rank
    H = inputs.device_normal((M, hidden), 1.0, base + 11, dev, torch.bfloat16)    # q, k, v, gate, up
    A = inputs.device_normal((M, hidden), 1.0, base + 12, dev, torch.bfloat16)    # o
    U = inputs.device_normal((M, mlp), 1.0, base + 13, dev, torch.bfloat16)       # down
    xs = {"q": H, "k": H, "v": H, "o": A, "gate": H, "up": H, "down": U}
    lins = [Linear(l, xs[l.name], dev, wl.seed + 100 * i, wl) for i, l in enumerate(wl.linears)]
    # adapter gradients as views of one flat fp32 buffer (one all-reduce per step)
    grads = FlatGrads([(l.lin.k_in, l.lin.n_out, wl.r) for l in lins], dev)
    for l, (dl1, dl2) in zip(lins, grads.views):
        l.dL1, l.dL2 = dl1, dl2
    return lins, grads, [H, A, U] + [l.dY for l in lins]


BWD_GROUPS = (("down",), ("gate", "up"), ("o",), ("q", "k", "v"))


def make_step(qlora, lins, grads, world, wl=WL, dropout=0.0):
    """One step; `ready(t)` (if given) is called before the step first reads input t.
    With `dropout` > 0 each linear applies LoRA dropout with its own keep mask.
    Without dropout the forward runs the linears that read the same input as
    one grouped call (q, k, v, gate and up on the layer input), in the order
    of their first use, and the backward as grouped calls in the order a
    layer's gradients arrive (BWD_GROUPS)."""
    groups, bwd_groups = [], []
    if dropout == 0:
        by_x = {}
        for l in lins:
            by_x.setdefault(l.X.data_ptr(), []).append(l)
        groups = [(g[0].X, qlora.FwdGroup([{"X": l.X, "q": l.q, "L1": l.L1, "L2": l.L2, "s": wl.s, "Y": l.Y,
                                             "T": l.T} for l in g])) for g in by_x.values()]
        # the backward as the layer's gradients arrive: down, then gate and up,
        # then o, then q, k and v
        by_name = {l.lin.name: l for l in lins}
        order = [[by_name[n] for n in names if n in by_name] for names in BWD_GROUPS]
        order = [g for g in order if g]
        rest = [l for l in reversed(lins) if all(l not in g for g in order)]
        order += [[l] for l in rest]
        bwd_groups = [([l.dY for l in g], qlora.BwdGroup(
            [{"dY": l.dY, "X": l.X, "T": l.T, "q": l.q, "L1": l.L1, "L2": l.L2, "s": wl.s, "dX": l.dX,
              "dL1": l.dL1, "dL2": l.dL2} for l in g], grad_dtype=torch.float32)) for g in order]

    def step(ready=None):
        for l in lins:
            l.q = qlora.quantize_nf4_dq(l.W, out=l.q)
        for X, grp in groups:
            if ready:
                ready(X)
            grp()
        for l in (lins if dropout > 0 else []):
            if ready:
                ready(l.X)
                if l.mask is not None:
                    ready(l.mask)
            qlora.linear_fwd(l.X, l.q, l.L1, l.L2, wl.s, Y=l.Y, T=l.T, dropout_mask=l.mask, dropout_p=dropout,
                             Xm=l.Xm)
        for dys, grp in bwd_groups:
            for t in (dys if ready else []):
                ready(t)
            grp()
        for l in (reversed(lins) if dropout > 0 else []):
            if ready:
                ready(l.dY)
            qlora.linear_bwd(l.dY, l.X, l.T, l.q, l.L1, l.L2, wl.s, grad_dtype=torch.float32,
                             dX=l.dX, dL1=l.dL1, dL2=l.dL2, dropout_mask=l.mask, dropout_p=dropout, Xm=l.Xm)
        grads.allreduce()
    return step


def run_e2e(args, step, flat, acts, dev, world, e0, e1, overlap=False):
    """Same step with host buffers: the step's activations and output gradients
    (`acts`, in the order the step first reads them) copied in from pinned host
    memory, adapter gradients copied out.  With `overlap`, the copies run on a
    copy stream and the step waits for each input just before it first reads
    it, so the transfers overlap quantization and the earlier linears."""
    pinned_in = [torch.empty(a.shape, dtype=a.dtype, pin_memory=True) for a in acts]
    for h, a in zip(pinned_in, acts):
        h.copy_(a)
    grads_host = torch.empty(flat.shape, dtype=flat.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in pinned_in)
    d2h = grads_host.numel() * grads_host.element_size()
    copy_stream = torch.cuda.Stream(dev)
    main = torch.cuda.current_stream(dev)

    def e2e_step():
        if not overlap:
            for h, a in zip(pinned_in, acts):
                a.copy_(h, non_blocking=True)
            step()
        else:
            # the copies may start once the previous step no longer reads the buffers
            copy_stream.wait_stream(main)
            done = {}
            with torch.cuda.stream(copy_stream):
                for h, a in zip(pinned_in, acts):
                    a.copy_(h, non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(copy_stream)
                    done[a.data_ptr()] = ev

            def ready(t):
                ev = done.pop(t.data_ptr(), None)
                if ev is not None:
                    main.wait_event(ev)
            step(ready)
            for ev in done.values():       # inputs the step never read still complete within it
                main.wait_event(ev)
        grads_host.copy_(flat, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0.record()
    for _ in range(args.steps):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    ms_e2e = e0.elapsed_time(e1) / args.steps
    t = torch.tensor([ms_e2e], device=dev)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    ms_e2e = float(t.item())

    return ms_e2e, h2d, d2h

TRAIN = {"llama7b-train": workloads.LLAMA7B_LAYER, "llama65b-train": workloads.LLAMA65B_LAYER,
         "llama33b-stack": workloads.LLAMA33B_STACK}


def train_config(args, wl, world):
    """The `config` of a training-workload line (both arms print the same one)."""
    return {"workload": wl.name + (f"[{args.linear} only]" if args.linear else "")
                        + (f"-lora-dropout{args.dropout:g}" if args.dropout > 0 else ""),
            "model": {"llama7b-train": "llama7b-layer-linears", "llama65b-train": "llama65b-layer-linears",
                      "llama33b-stack": "llama33b-8-layer-stack"}[args.workload],
            "global_batch": (16 if wl.M == 8192 and args.workload == "llama7b-train" else 4) * world,
            "seq_len": 512 if args.workload == "llama7b-train" else 2048,
            "tokens_per_rank": wl.M, "lora_r": wl.r, "lora_alpha": wl.alpha, "layers": wl.layers,
            "parallelism": f"dp{world}" if world > 1 else "single",
            "step": f"quantize {7 * wl.layers} fp32 weights to NF4+DQ, fwd + bwd of the "
                    f"{7 * wl.layers} QLoRA linears"
                    + (" (forward of the linears that read the same input as one grouped call: q, k, v, "
                       "gate, up on the layer input; backward grouped as the gradients arrive: down, "
                       "{gate, up}, o, {q, k, v})" if wl.layers == 1 and args.dropout == 0 else "")
                    + (" (layer to layer: H' = bf16(down(up(H)) + R); each layer's six linears on H as one "
                       "grouped forward and one grouped backward)" if wl.layers > 1 else "")
                    + (", all-reduce of adapter grads" if world > 1 else "")
                    + (f", LoRA dropout p = {args.dropout:g} on every adapter (one seeded keep mask per "
                       f"linear, copied in with the inputs in e2e)" if args.dropout > 0 else ""),
            "l2": "inputs larger than L2 (>1 GB touched per step), no flush"}


def run_ours(args, rank, world, local_rank):
    import bit_nf4_quantized_02_b200 as qlora
    from bit_nf4_quantized_02_b200 import _lib

    _lib.load()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = TRAIN[args.workload]
    if wl.layers > 1 and args.dropout > 0:
        raise SystemExit("bench.py: --dropout applies to the single-layer training workloads")
    if wl.layers > 1:
        from bit_nf4_quantized_02_b200.stack import QLoRAStack, SEEDED_DY
        hidden, mlp = wl.linears[0].n_out, wl.linears[4].n_out
        st = QLoRAStack(qlora, hidden, mlp, wl.layers, wl.M, wl.r, wl.alpha, wl.seed + 100_000 * rank, dev,
                        lambda shape, std, seed, dtype: inputs.device_normal(shape, std, seed, dev, dtype))
        st.quantize()     # allocate the quantized buffers once
        grads, flat = st.grads, st.grads.flat
        acts = [st.H[0], st.dH[-1]] + st.R + [st.lin[l][n].dY for l in range(wl.layers) for n in SEEDED_DY]
        step = st.step
        sel = wl.linears * wl.layers
    else:
        lins, grads, acts = build_layer(dev, rank, wl)
        if args.dropout > 0:
            for i, l in enumerate(lins):
                l.mask = device_dropout_mask(wl.M, l.lin.k_in, args.dropout, wl.seed + 1000 * rank + 50 + i, dev)
                l.Xm = torch.empty_like(l.X)
        # copy order for the end-to-end run: the step's first read of each input
        # (with dropout each linear's keep mask right after its input)
        if args.dropout > 0:
            first = []
            for l in lins:
                if all(l.X.data_ptr() != a.data_ptr() for a in first):
                    first.append(l.X)
                first.append(l.mask)
            acts = first + acts[3:][::-1]
        else:
            acts = acts[:3] + acts[3:][::-1]
        flat = grads.flat
        if args.linear:
            lins = [l for l in lins if l.lin.name == args.linear]
        for l in lins:  # allocate the quantized buffers once
            l.q = qlora.quantize_nf4_dq(l.W)
        step = make_step(qlora, lins, grads, world, wl, dropout=args.dropout)
        sel = [l.lin for l in lins]
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if qlora.last_device_error() != 0:
        raise RuntimeError("device error during warm-up")

    # The per-launch event log (kernel table, roofline) comes from its own pass
    # of the same steps on every rank, ahead of the timed pass: events between
    # launches would serialise the programmatic dependent launches there.  A
    # pause after it lets the GPU leave the power state the pass drove it to.
    qlora.profile_start(args.steps * 200 * wl.layers + 64)
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    launches = qlora.profile_stop()
    time.sleep(1.0)

    sampler = ClockSampler(list(range(world)) if world > 1 else [local_rank]) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.5)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop() if sampler else None
    ms = e0.elapsed_time(e1) / args.steps
    t = torch.tensor([ms], device=dev)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    ms = float(t.item())
    if qlora.last_device_error() != 0:
        raise RuntimeError("device error during the timed region")

    # ---------------- end to end: host inputs in, adapter gradients out
    if args.no_e2e:
        ms_e2e, h2d, d2h = None, None, None
    else:
        ms_e2e, h2d, d2h = run_e2e(args, step, flat, acts, dev, world, e0, e1, overlap=wl.layers == 1)

    if rank != 0:
        return None
    flops = step_flops(sel, wl.M, wl.r) * world
    value = flops / (ms * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    # dominant kernel: the tcgen05 GEMM launches of the Y and dX products
    per_kind = {}
    for kind, kms in launches:
        c = per_kind.setdefault(kind, [0, 0.0])
        c[0] += 1
        c[1] += kms
    dom_ms = per_kind.get("gemm_Y", [0, 0.0])[1] + per_kind.get("gemm_dX", [0, 0.0])[1]
    dom_n = per_kind.get("gemm_Y", [0, 0.0])[0] + per_kind.get("gemm_dX", [0, 0.0])[0]
    # with LoRA dropout dX's adapter term runs as its own product (gemm_Z),
    # so the dX launches do the base product alone
    dom_flops = args.steps * sum(linear_flops(wl.M, l.n_out, l.k_in, wl.r)["gemm_Y"] +
                                 linear_flops(wl.M, l.n_out, l.k_in, wl.r)["gemm_dX"]
                                 - (2 * wl.M * wl.r * l.k_in if args.dropout > 0 else 0) for l in sel)
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12 if dom_ms > 0 else None
    # The burst GEMM peak while the SM clock held its maximum through the timed
    # region; the sustained (power-capped) one once the clock dropped.
    at_max = bool(clocks and clocks.get("sm_mhz") and clocks.get("sm_max_mhz")
                  and clocks["sm_mhz"] >= 0.97 * clocks["sm_max_mhz"]
                  and "sw_power_cap" not in (clocks.get("reasons") or []))
    peak_key = "bf16_tflops" if at_max else "bf16_tflops_sustained"
    peak = peaks.get(peak_key, FALLBACK_PEAKS[peak_key])
    # DRAM traffic per launch: the ncu-measured ratio of DRAM bytes to algorithmic
    # bytes for these launches (captured at the q shape), applied to the average
    # algorithmic bytes of the timed launches; null once the kernel source changed.
    traffic = None
    tp = os.path.join(ROOT, "profiles", "tc_gemm_traffic.txt")
    if os.path.exists(tp):
        with open(tp) as f:
            tr = json.load(f)
        if tr.get("source_hash") == source_hash("tc_gemm.cuh", "common.cuh"):
            M, r = wl.M, wl.r
            alg = [2 * M * l.k_in + 2 * l.n_out * l.k_in + 2 * M * l.n_out + 2 * M * r + 2 * r * l.n_out for l in sel]
            alg += [2 * M * l.n_out + 2 * l.n_out * l.k_in + 2 * M * l.k_in + 2 * M * r + 2 * r * l.k_in for l in sel]
            traffic = tr["traffic_over_algorithmic"] * sum(alg) / len(alg)
    total_kernel_ms = sum(v[1] for v in per_kind.values())
    kernels = {k: {"launches_per_step": v[0] / args.steps, "ms_per_step": v[1] / args.steps,
                   "share": v[1] / total_kernel_ms if total_kernel_ms else None}
               for k, v in sorted(per_kind.items(), key=lambda kv: -kv[1][1])}
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": train_config(args, wl, world),
        "e2e": ({"value": flops / (ms_e2e * 1e-3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": h2d,
                 "d2h_bytes_per_step": d2h,
                 "copies": ("host->device copies on a copy stream in the order the step first reads them, "
                            "overlapping quantization and compute" if wl.layers == 1 else
                            "host->device copies before the step")} if ms_e2e else None),
        "gpu_launches": _kernel_count(launches),
        "roofline": {"bound": "tensor", "kernel": "tc_gemm (Y = X W^T + T L2 and dX = dY W + G L1^T)",
                     "traffic_unit": "bytes per launch (DRAM read + write)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak if achieved else None, "traffic": traffic,
                     "peak_source": f"{peak_src} {peak_key}",
                     "launches_timed": dom_n, "avg_launch_ms": dom_ms / dom_n if dom_n else None},
        "kernels": kernels,
        "clocks": clocks,
    }
    default_line = world == 1 and not args.linear and args.workload == "llama7b-train" and args.dropout == 0
    if default_line and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline()
    if default_line and not args.no_subrecords:
        # the other targets, each timed on its own (CUDA events) after the headline:
        # the decode-sized forward (LLaMA-65B layer at 16 tokens) and the quantizer
        del lins, grads, acts, step, flat
        torch.cuda.empty_cache()
        out["decode"] = decode_subrecord(args, rank, world, local_rank)
        torch.cuda.empty_cache()
        out["quantizer"] = quantizer_subrecord(args, rank, world, local_rank)
    return out


# --------------------------------------------------------------------------- other workloads
def _timed(qlora, step, args, dev, world, rank, local_rank, profile=True):
    """Warm up, then time args.steps steps with CUDA events (max over ranks)."""
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if qlora.last_device_error() != 0:
        raise RuntimeError("device error during warm-up")
    # The per-launch event log (kernel table, roofline) comes from its own pass
    # of the same steps, ahead of the timed pass: events between launches
    # would serialise the programmatic dependent launches there.  A pause
    # after it lets the GPU leave the power state the pass drove it to.
    launches = []
    if profile:
        qlora.profile_start(args.steps * 256 + 64)
        for _ in range(args.steps):
            step()
        torch.cuda.synchronize()
        launches = qlora.profile_stop()
        time.sleep(1.0)
    sampler = ClockSampler([local_rank]) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.5)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    ms = e0.elapsed_time(e1) / args.steps
    t = torch.tensor([ms], device=dev)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    if qlora.last_device_error() != 0:
        raise RuntimeError("device error during the timed region")
    return float(t.item()), launches, clocks


def _kernel_table(launches, steps):
    per_kind = {}
    for kind, kms in launches:
        c = per_kind.setdefault(kind, [0, 0.0])
        c[0] += 1
        c[1] += kms
    total = sum(v[1] for v in per_kind.values())
    return per_kind, {k: {"launches_per_step": v[0] / steps, "ms_per_step": v[1] / steps,
                          "share": v[1] / total if total else None}
                      for k, v in sorted(per_kind.items(), key=lambda kv: -kv[1][1])}


# Kernels behind one entry of the library's event log: the few-token forward
# logs its chain (T accumulation, product, epilogue) as one entry.
KERNELS_PER_ENTRY = {"fused_fwd": 3}


def _kernel_count(launches) -> int:
    return sum(KERNELS_PER_ENTRY.get(kind, 1) for kind, _ in launches)


def _graph_ms(step, dev, steps):
    """Per-step ms of ``step`` captured once in a CUDA graph and replayed."""
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        step()
        with torch.cuda.graph(g, stream=side):
            step()
    torch.cuda.current_stream(dev).wait_stream(side)
    for _ in range(3):
        g.replay()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def _eager_ms(step, steps):
    for _ in range(3):
        step()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def run_decode(args, rank, world, local_rank):
    """LLaMA-65B layer forward at 16 tokens: the memory-bound few-token path.

    The seven projections run as the layer's data flow allows: q, k, v, gate
    and up (which all read the layer input H) as one grouped call, then o
    (reads the attention output A) and down (reads U).  The line also reports
    the same step as seven single-linear calls and as one group of all seven.
    """
    import bit_nf4_quantized_02_b200 as qlora
    wl = workloads.LLAMA65B_LAYER
    M, r, s = args.tokens or wl.extra["M_decode"], wl.r, wl.s
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    base = wl.seed + 1000 * rank
    H = inputs.device_normal((M, 8192), 1.0, base + 1, dev, torch.bfloat16)
    A = inputs.device_normal((M, 8192), 1.0, base + 2, dev, torch.bfloat16)
    U = inputs.device_normal((M, 22016), 1.0, base + 3, dev, torch.bfloat16)
    xs = {"q": H, "k": H, "v": H, "o": A, "gate": H, "up": H, "down": U}
    lins, members = [], {}
    nbytes = 0
    for i, lin in enumerate(wl.linears):
        N, K = lin.n_out, lin.k_in
        W = inputs.device_normal((N, K), inputs.WEIGHT_STD, wl.seed + 100 * i, dev)
        q = qlora.quantize_nf4_dq(W)
        del W
        L1 = inputs.device_normal((K, r), 1.0 / np.sqrt(K), wl.seed + 100 * i + 1, dev, torch.bfloat16)
        L2 = inputs.device_normal((r, N), inputs.L2_STD, wl.seed + 100 * i + 2, dev, torch.bfloat16)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        T = torch.empty(M, 2 * r, dtype=torch.bfloat16, device=dev)
        lins.append((xs[lin.name], q, L1, L2, Y, T))
        members[lin.name] = {"X": xs[lin.name], "q": q, "L1": L1, "L2": L2, "s": s, "Y": Y, "T": T}
        # algorithmic bytes: NF4+DQ weight, LoRA factors, X read, Y and T written
        nbytes += q.nbytes() + 2 * r * (K + N) + 2 * M * K + 2 * M * N + 2 * M * 2 * r
    torch.cuda.synchronize()
    # grouped calls with their arguments marshalled once (qlora.FwdGroup)
    groups = [qlora.FwdGroup([members[n] for n in ("q", "k", "v", "gate", "up")]),
              qlora.FwdGroup([members["o"]]), qlora.FwdGroup([members["down"]])]
    everything = qlora.FwdGroup([members[l.name] for l in wl.linears])

    def step():                       # the layer's data flow: three grouped calls
        for grp in groups:
            grp()

    def step_single():                # seven single-linear calls
        for X, q, L1, L2, Y, T in lins:
            qlora.linear_fwd(X, q, L1, L2, s, Y=Y, T=T)

    def step_one_group():             # all seven in one launch chain
        everything()

    ms, launches, clocks = _timed(qlora, step, args, dev, world, rank, local_rank)
    ms_graph = _graph_ms(step, dev, args.steps)
    variants = {}
    for name, fn in (("seven_single_calls", step_single), ("one_group_of_seven", step_one_group)):
        e, gms = _eager_ms(fn, args.steps), _graph_ms(fn, dev, args.steps)
        variants[name] = {"ms_per_step": e, "value": nbytes / (e * 1e-3) / 1e9, "graph_ms_per_step": gms,
                          "graph_value": nbytes / (gms * 1e-3) / 1e9}
    if qlora.last_device_error() != 0:
        raise RuntimeError("device error in the decode variants")
    if rank != 0:
        return None
    peaks, peak_src = load_peaks()
    per_kind, kernels = _kernel_table(launches, args.steps)
    dom = per_kind.get("fused_fwd") or [0, 0.0]
    achieved = nbytes * args.steps / (dom[1] * 1e-3) / 1e9 if dom[1] > 0 else None
    peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    for v in variants.values():
        v["unit"] = "GB/s"
        v["graph_frac_of_hbm"] = v["graph_value"] / peak
    return {
        "metric": "QLoRA NF4 linear forward, NF4-weight-bound GB/s", "value": nbytes * world / (ms * 1e-3) / 1e9,
        "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"llama65b-layer-7-linears-forward-M{M}-r64", "tokens": M, "lora_r": r,
                   "bytes_per_step": nbytes, "l2": "weights (418 MB) larger than L2, no flush",
                   "step": "forward of the 7 QLoRA linears (weights resident, quantized once) as the layer's "
                           "data flow groups them: {q, k, v, gate, up} on H, then o on A, then down on U"},
        "graph": {"ms_per_step": ms_graph, "value": nbytes * world / (ms_graph * 1e-3) / 1e9, "unit": "GB/s",
                  "frac_of_hbm": nbytes / (ms_graph * 1e-3) / 1e9 / peak},
        "variants": variants,
        "gpu_launches": _kernel_count(launches),
        "roofline": {"bound": "hbm", "kernel": ("few-token forward chain (lora_down_small + " +
                                                "nf4_decode_fwd: weight decoded into TMEM, tcgen05" + " + epilogue)"),
                     "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak if achieved else None, "traffic": None,
                     "peak_source": f"{peak_src} hbm_gbs", "launches_timed": dom[0],
                     "avg_launch_ms": dom[1] / dom[0] if dom[0] else None},
        "kernels": kernels, "clocks": clocks,
    }


def run_quantizer(args, rank, world, local_rank):
    """NF4 + DQ quantize, then dequantize, of the LLaMA-7B-shaped bf16 weights (with outliers)."""
    import bit_nf4_quantized_02_b200 as qlora
    wl = workloads.QUANTIZER_7B
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    mats = []
    nbytes_q = nbytes_d = 0
    for i, lin in enumerate(wl.linears):
        W = inputs.device_weight_with_outliers(lin.n_out, lin.k_in, wl.seed + 1000 * rank + i, dev)
        q = qlora.quantize_nf4_dq(W, table=args.table)
        out = torch.empty_like(W)
        mats.append((W, q, out))
        nbytes_q += W.numel() * 2 + q.nbytes()
        nbytes_d += q.nbytes() + W.numel() * 2
    torch.cuda.synchronize()

    def step():
        for W, q, out in mats:
            qlora.quantize_nf4_dq(W, out=q, table=args.table)
        for W, q, out in mats:
            qlora.dequant(q, out=out)

    ms, launches, clocks = _timed(qlora, step, args, dev, world, rank, local_rank)
    # the same step replayed from a CUDA graph: the launches without the host's per-call cost
    ms_graph = _graph_ms(step, dev, args.steps)
    if qlora.last_device_error() != 0:
        raise RuntimeError("device error in the graph replay of the quantizer step")
    if rank != 0:
        return None
    # Accuracy of the storage format (outside the timed region): RMS error of
    # the dequantized weights against the originals, relative to their RMS,
    # for both code tables on the same weights (the comparison of §4).
    accuracy = {}
    for t in ("nf4", "fp4"):
        se = sq = 0.0
        for W, _, _ in mats:
            wh = qlora.dequant(qlora.quantize_nf4_dq(W, table=t)).float()
            se += float((wh - W.float()).square().sum())
            sq += float(W.float().square().sum())
        accuracy[f"{t}_rel_rms_error"] = (se / sq) ** 0.5
    peaks, peak_src = load_peaks()
    per_kind, kernels = _kernel_table(launches, args.steps)
    peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    qk, dk = per_kind.get("quantize", [0, 0.0]), per_kind.get("dequant", [0, 0.0])
    dq = per_kind.get("dq_constants", [0, 0.0])
    q_ms = qk[1] + dq[1]
    roof_q = nbytes_q * args.steps / (q_ms * 1e-3) / 1e9 if q_ms else None
    roof_d = nbytes_d * args.steps / (dk[1] * 1e-3) / 1e9 if dk[1] else None
    return {
        "metric": ("NF4" if args.table == "nf4" else "FP4 (E2M1)") + "+DQ quantize + dequantize GB/s", "value": (nbytes_q + nbytes_d) * world / (ms * 1e-3) / 1e9,
        "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u8", "data": "synthetic",
        "config": {"workload": wl.name + ("" if args.table == "nf4" else "-fp4"),
                   "code_table": args.table, "params": sum(l.n_out * l.k_in for l in wl.linears),
                   "bytes_quantize": nbytes_q, "bytes_dequant": nbytes_d,
                   "l2": "weights (667 MB bf16) larger than L2, no flush"},
        "gpu_launches": _kernel_count(launches),
        "graph": {"ms_per_step": ms_graph, "value": (nbytes_q + nbytes_d) * world / (ms_graph * 1e-3) / 1e9,
                  "unit": "GB/s", "frac_of_hbm": (nbytes_q + nbytes_d) / (ms_graph * 1e-3) / 1e9
                  / load_peaks()[0].get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])},
        "roofline": {"bound": "hbm", "kernel": "quantize (K1 + K2) and dequant (K3)",
                     "achieved": roof_q, "achieved_dequant": roof_d, "peak": peak, "unit": "GB/s",
                     "frac": roof_q / peak if roof_q else None, "frac_dequant": roof_d / peak if roof_d else None,
                     "traffic": None, "peak_source": f"{peak_src} hbm_gbs"},
        "accuracy": accuracy,
        "kernels": kernels, "clocks": clocks,
    }


# --------------------------------------------------------------------------- sub-records
def _subargs(args, **kw):
    ns = argparse.Namespace(**vars(args))
    ns.__dict__.update(kw)
    return ns


SUB_KEYS = ("metric", "value", "unit", "ms_per_step", "steps", "warmup", "config", "graph", "variants",
            "roofline", "accuracy", "kernels", "gpu_launches", "clocks")


def decode_subrecord(args, rank, world, local_rank):
    """Config 4a in the default line: the LLaMA-65B layer forward at 16 tokens."""
    sub = run_decode(_subargs(args, steps=20, warmup=3, tokens=workloads.LLAMA65B_LAYER.extra["M_decode"]),
                     rank, world, local_rank)
    rec = {k: sub[k] for k in SUB_KEYS if k in sub}
    peak = sub["roofline"]["peak"]
    rec["frac_of_hbm"] = sub["value"] / peak
    if not args.no_cpu_baseline:
        rec["cpu_baseline"] = decode_cpu_baseline()
    return rec


def quantizer_subrecord(args, rank, world, local_rank):
    """Config 3 in the default line: NF4 + DQ quantize and dequantize of LLaMA-7B-shaped bf16 weights."""
    sub = run_quantizer(_subargs(args, steps=20, warmup=3, table="nf4"), rank, world, local_rank)
    rec = {k: sub[k] for k in SUB_KEYS if k in sub}
    peak = sub["roofline"]["peak"]
    rec["frac_of_hbm"] = sub["value"] / peak
    if not args.no_cpu_baseline:
        rec["cpu_baseline"] = quantizer_cpu_baseline()
    return rec


def nf4_nbytes(n_out: int, k_in: int) -> int:
    """Bytes of a weight in the stored NF4 + DQ format (codes, E4M3 block codes, c1, mean)."""
    n = n_out * k_in
    nblk = (n + 63) // 64
    return (n + 1) // 2 + nblk + 4 * ((nblk + 255) // 256) + 4


def decode_step_bytes(M: int, r: int) -> int:
    """Algorithmic bytes of the decode step: NF4 + DQ weights, LoRA factors, X read, Y and T written."""
    return sum(nf4_nbytes(l.n_out, l.k_in) + 2 * r * (l.k_in + l.n_out) + 2 * M * l.k_in + 2 * M * l.n_out
               + 2 * M * 2 * r for l in workloads.LLAMA65B_LAYER.linears)


DECODE_SAMPLE = 8


def decode_cpu_baseline():
    """The oracle's doubleDequant + fp64 forward on 1/8 of each LLaMA-65B linear's
    output rows at 16 tokens (the weights quantized beforehand, untimed), scaled x8."""
    from oracle import nf4dq, qlora_linear
    wl = workloads.LLAMA65B_LAYER
    M, r, s = wl.extra["M_decode"], wl.r, wl.s
    g = inputs.rng(wl.seed + 9)
    data = []
    for lin in wl.linears:
        N, K = lin.n_out, lin.k_in
        rows = N // DECODE_SAMPLE
        oq = nf4dq.quantize_nf4_dq(inputs.weight_f32(g, rows, K))
        L1, L2 = inputs.lora_factors(g, K, rows, r)
        data.append((oq, inputs.normal_bf16(g, (M, K)).float().numpy().astype(np.float64),
                     L1.float().numpy().astype(np.float64), L2.float().numpy().astype(np.float64)))
    t0 = time.perf_counter()
    for oq, X, L1, L2 in data:
        qlora_linear.forward(X, nf4dq.dequantize(oq), L1, L2, s)
    dt = time.perf_counter() - t0
    return {"value": decode_step_bytes(M, r) / (dt * DECODE_SAMPLE) / 1e9, "unit": "GB/s", "cores": _cores(),
            "kind": "oracle", "sample_seconds": dt,
            "sample": f"doubleDequant + fp64 forward of 1/{DECODE_SAMPLE} of each linear's output rows at {M} "
                      f"tokens (weights quantized beforehand); full-step time = {DECODE_SAMPLE} x sample"}


QUANT_SAMPLE = 8


def quantizer_cpu_baseline():
    """The oracle's NF4 + DQ quantize and doubleDequant of 1/8 of each matrix's rows, scaled x8."""
    from oracle import nf4dq
    wl = workloads.QUANTIZER_7B
    g = inputs.rng(wl.seed + 9)
    mats = [inputs.weight_bf16_with_outliers(g, l.n_out // QUANT_SAMPLE, l.k_in).float().numpy()
            for l in wl.linears]
    t0 = time.perf_counter()
    for W in mats:
        nf4dq.dequantize(nf4dq.quantize_nf4_dq(W))
    dt = time.perf_counter() - t0
    nbytes = sum(2 * (2 * l.n_out * l.k_in + nf4_nbytes(l.n_out, l.k_in)) for l in wl.linears)
    return {"value": nbytes / (dt * QUANT_SAMPLE) / 1e9, "unit": "GB/s", "cores": _cores(), "kind": "oracle",
            "sample_seconds": dt,
            "sample": f"NF4+DQ quantize and doubleDequant of 1/{QUANT_SAMPLE} of each matrix's rows; "
                      f"full-step time = {QUANT_SAMPLE} x sample"}


# --------------------------------------------------------------------------- oracle timing
SAMPLE_SLICE = 64   # the CPU sample is 1/64 of a step: 128 of the 8192 tokens, 1/64 of each weight's rows


def _oracle_sample_setup():
    g = inputs.rng(WL.seed + 7)
    Ms = WL.M // SAMPLE_SLICE
    data = []
    for lin in WL.linears:
        N, K = lin.n_out, lin.k_in
        rows = N // SAMPLE_SLICE
        data.append({
            "W_rows": inputs.weight_f32(g, rows, K),
            # a seeded stand-in for the dequantized weight (the oracle's cost does not depend on values)
            "W_hat": inputs.normal_bf16(g, (N, K), 0.02).float().numpy(),
            "X": inputs.normal_bf16(g, (Ms, K)).float().numpy(),
            "dY": inputs.normal_bf16(g, (Ms, N)).float().numpy(),
            "L1": inputs.normal_bf16(g, (K, WL.r), 1 / np.sqrt(K)).float().numpy(),
            "L2": inputs.normal_bf16(g, (WL.r, N), 0.01).float().numpy(),
        })
    return data


def _oracle_sample_step(data):
    from oracle import nf4dq, qlora_linear
    for d in data:
        nf4dq.quantize_nf4_dq(d["W_rows"])
        qlora_linear.forward(d["X"], d["W_hat"], d["L1"], d["L2"], WL.s)
    for d in reversed(data):
        qlora_linear.backward(d["dY"], d["X"], d["W_hat"], d["L1"], d["L2"], WL.s)


def _cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


SAMPLE_DESC = (f"1/{SAMPLE_SLICE} of a step: NF4+DQ of 1/{SAMPLE_SLICE} of each weight's rows and fp64 fwd+bwd "
               f"of the 7 linears at {WL.M // SAMPLE_SLICE} of {WL.M} tokens; full-step time = {SAMPLE_SLICE} x sample")


def cpu_baseline(reps=1):
    """The oracle on the host cores (all BLAS threads), and again on one thread."""
    data = _oracle_sample_setup()
    t0 = time.perf_counter()
    for _ in range(reps):
        _oracle_sample_step(data)
    dt = (time.perf_counter() - t0) / reps
    step_s = dt * SAMPLE_SLICE
    out = {"value": step_flops() / step_s / 1e12, "unit": UNIT, "cores": _cores(), "kind": "oracle",
           "sample": SAMPLE_DESC, "sample_seconds": dt}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            t0 = time.perf_counter()
            _oracle_sample_step(data)
            dt1 = time.perf_counter() - t0
        out["single_thread"] = {"value": step_flops() / (dt1 * SAMPLE_SLICE) / 1e12, "unit": UNIT, "cores": 1,
                                "sample_seconds": dt1}
    except ImportError:
        pass
    return out


def run_reference(args, rank, world):
    if rank != 0:
        return None
    data = _oracle_sample_setup()
    for _ in range(args.warmup):
        _oracle_sample_step(data)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_sample_step(data)
    dt = (time.perf_counter() - t0) / args.steps
    step_s = dt * SAMPLE_SLICE
    value = step_flops() / step_s / 1e12
    cores = _cores()
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "step_is_sample": f"each timed step is the 1/{SAMPLE_SLICE} sample below, so ms_per_step is the sample's "
                          f"time; value = the sample's FLOPs / that time (full-step time {step_s * 1e3:.0f} ms)",
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": train_config(_subargs(args, workload="llama7b-train", linear=None, dropout=0.0), WL, 1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": SAMPLE_DESC,
                         "sample_seconds": dt},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_cublas_compare(args, rank, world, local_rank):
    """Context for the GEMM roofline: the library's Y and dX products (X W_hat^T
    + T_hi L2 and dY W_hat + G_hi L1^T, event log of linear_fwd / linear_bwd)
    against cuBLAS (torch.mm, bf16 in, fp32 accumulate, bf16 out) on the same
    LLaMA-7B shapes at 8192 tokens."""
    import bit_nf4_quantized_02_b200 as qlora
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = WL
    M, r, s = wl.M, wl.r, wl.s
    rows = []
    seen = set()
    for i, lin in enumerate(wl.linears):
        N, K = lin.n_out, lin.k_in
        if (N, K) in seen:
            continue
        seen.add((N, K))
        X = inputs.device_normal((M, K), 1.0, wl.seed + 7 * i, dev, torch.bfloat16)
        W = inputs.device_normal((N, K), inputs.WEIGHT_STD, wl.seed + 7 * i + 1, dev)
        q = qlora.quantize_nf4_dq(W)
        Wb = qlora.dequant(q)
        L1 = inputs.device_normal((K, r), 1.0 / np.sqrt(K), wl.seed + 7 * i + 2, dev, torch.bfloat16)
        L2 = inputs.device_normal((r, N), inputs.L2_STD, wl.seed + 7 * i + 3, dev, torch.bfloat16)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        T = torch.empty(M, 2 * r, dtype=torch.bfloat16, device=dev)
        for _ in range(args.warmup):
            qlora.linear_fwd(X, q, L1, L2, s, Y=Y, T=T)
            torch.mm(X, Wb.t(), out=Y)
        torch.cuda.synchronize()
        dY = inputs.device_normal((M, N), 1.0, wl.seed + 7 * i + 4, dev, torch.bfloat16)
        dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
        for _ in range(args.warmup):
            qlora.linear_bwd(dY, X, T, q, L1, L2, s, dX=dX)
            torch.mm(dY, Wb, out=dX)
        torch.cuda.synchronize()
        qlora.profile_start(args.steps * 16 + 16)
        for _ in range(args.steps):
            qlora.linear_fwd(X, q, L1, L2, s, Y=Y, T=T)
            qlora.linear_bwd(dY, X, T, q, L1, L2, s, dX=dX)
        torch.cuda.synchronize()
        log = qlora.profile_stop()
        ours = [ms for kind, ms in log if kind == "gemm_Y"]
        ours_dx = [ms for kind, ms in log if kind == "gemm_dX"]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        warm, cold, warm_dx, cold_dx = [], [], [], []
        for _ in range(args.steps):
            for lst, fl, fn in ((warm, False, lambda: torch.mm(X, Wb.t(), out=Y)),
                                (cold, True, lambda: torch.mm(X, Wb.t(), out=Y)),
                                (warm_dx, False, lambda: torch.mm(dY, Wb, out=dX)),
                                (cold_dx, True, lambda: torch.mm(dY, Wb, out=dX))):
                if fl:
                    flush.fill_(1)    # evict the operands from L2 (256 MB written)
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize()
                lst.append(e0.elapsed_time(e1))
        f_ours = linear_flops(M, N, K, r)["gemm_Y"]
        f_mm = 2 * M * N * K
        rows.append({"shape": f"{M}x{N}x{K}", "linears": [l.name for l in wl.linears if (l.n_out, l.k_in) == (N, K)],
                     "ours_gemm_Y_ms": statistics.median(ours), "ours_tflops": f_ours / statistics.median(ours) / 1e9,
                     "cublas_mm_ms_l2_warm": statistics.median(warm),
                     "cublas_tflops_l2_warm": f_mm / statistics.median(warm) / 1e9,
                     "cublas_mm_ms_l2_flushed": statistics.median(cold),
                     "cublas_tflops_l2_flushed": f_mm / statistics.median(cold) / 1e9,
                     "ours_gemm_dX_ms": statistics.median(ours_dx),
                     "ours_dx_tflops": linear_flops(M, N, K, r)["gemm_dX"] / statistics.median(ours_dx) / 1e9,
                     "cublas_dx_tflops_l2_warm": f_mm / statistics.median(warm_dx) / 1e9,
                     "cublas_dx_tflops_l2_flushed": f_mm / statistics.median(cold_dx) / 1e9})
        del flush, dY, dX
        del X, W, q, Wb, L1, L2, Y, T
    peaks, src = load_peaks()
    return {"metric": "Y product TFLOP/s, library tcgen05 GEMM against cuBLAS on the same shapes", "unit": "TFLOP/s",
            "rows": rows, "peak_bf16_tflops": peaks.get("bf16_tflops"), "peak_source": src,
            "note": "median over --steps single calls; the library's time is its event-log time of the Y launch "
                    "inside linear_fwd, right after the dequant and T launches (which also adds T_hi L2 as 2 M r N "
                    "more FLOPs); cuBLAS via torch.mm on the dequantized weight, timed back to back (L2 warm) and "
                    "after writing 256 MB (L2 flushed)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) measurement")
    ap.add_argument("--no-subrecords", action="store_true",
                    help="default workload: skip the decode (16-token) and quantizer sub-records")
    ap.add_argument("--table", choices=["nf4", "fp4"], default="nf4",
                    help="4-bit code table of the quantizer workload (fp4: FP4 E2M1, compared against NF4)")
    ap.add_argument("--dropout", type=float, default=0.0,
                    help="LoRA dropout probability on every adapter (single-layer training workloads)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="llama65b-decode: tokens per step (default 16; 33..128 run the tcgen05 fused forward)")
    ap.add_argument("--cublas-compare", action="store_true",
                    help="print the library's Y GEMM against cuBLAS (torch.mm) on the LLaMA-7B shapes, then exit")
    ap.add_argument("--linear", choices=[l.name for l in WL.linears], default=None,
                    help="restrict the step to one linear of the layer (profiling runs)")
    ap.add_argument("--workload", choices=list(TRAIN) + ["llama65b-decode", "quantizer"], default="llama7b-train",
                    help="llama7b-train (default, the headline): quantize + fwd + bwd of a LLaMA-7B layer at 8192 "
                         "tokens; llama65b-train: the same for a LLaMA-65B layer at 4x2048 tokens; llama33b-stack: "
                         "eight LLaMA-33B layers at 4x2048 tokens, forward then backward; llama65b-decode: forward "
                         "of a LLaMA-65B layer at 16 tokens; quantizer: NF4+DQ quantize and dequantize of "
                         "LLaMA-7B-shaped bf16 weights")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        out = run_reference(args, rank, world)
    else:
        if world > 1:
            torch.cuda.set_device(local_rank)
            torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                                 device_id=torch.device("cuda", local_rank))
        try:
            if args.cublas_compare:
                out = run_cublas_compare(args, rank, world, local_rank)
            elif args.workload == "llama65b-decode":
                out = run_decode(args, rank, world, local_rank)
            elif args.workload == "quantizer":
                out = run_quantizer(args, rank, world, local_rank)
            else:
                out = run_ours(args, rank, world, local_rank)
        finally:
            if world > 1:
                torch.distributed.destroy_process_group()
    if out is not None and rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
