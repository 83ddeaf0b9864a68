#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--layers L] [--no-extras] [--no-e2e] [--no-cpu]
    python bench.py --case WORKLOAD [--linear J] [--tokens M] [--iters I] [--fwd-only]
    python bench.py --cpu-configs

Headline workload (default, ``stack_65b``): the 65B-shaped decoder stack, 80
layers x 7 linears (q, k, v, o 8192 x 8192; gate, up 22016 x 8192; down
8192 x 22016), every W ~ N(0, 0.015^2) quantised once to NF4 (blocksize 64)
with double-quantised scales (256) and kept resident (33.4 GB); LoRA r = 64,
alpha = 16 on every linear; 4 x 512 = 2048 tokens per GPU.  One step is the
forward pass of all 560 linears in layer order followed by the backward pass
(dX, dA, dB) in reverse order.  The metric counts fwd + bwd FLOPs
(4MNK + 6Mr(N + K) per linear).  The layers have no attention or activation
between them: every linear position reads its own seeded N(0, 1) activations
of its input width, shared by the 80 layers.

With N > 1 (torchrun, one process per GPU) every rank holds the same frozen
stack and its own 2048 tokens; each layer's LoRA gradients (one flat buffer
per layer) are summed over ranks by an NCCL all-reduce started right after
that layer's backward, so that it runs beside the backward of the layer
below (data parallelism; weak scaling).  Rank 0 prints one JSON line.

At one GPU the line also carries the other workloads as extra keys: the
whole 7B stack (32 x 7 linears, r = 16), the 7B attention projection with
quantisation inside the step, the 7B MLP at 8192 tokens, decode-sized
batches (M = 1, 16) and the adapter merge.

--impl reference times the CPU oracle (oracle/) on the host cores on a
bounded sample of the same workload.  --case runs one linear of a workload
for single-kernel profiles.  --cpu-configs times the oracle on every
configuration (long; for the baseline table).
"""

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = "stack_65b"
METRIC = "QLoRA linear fwd+bwd TFLOP/s and NF4 weight GB/s at 1 B200; % of roofline"
UNIT = "TFLOP/s"
STACK_TOKENS = 2048
CPU_SAMPLE_TOKENS = 64  # tokens of the oracle's bounded sample on the stacks


def fwd_flops(M, N, K, r):
    return 2 * M * N * K + 2 * M * K * r + 2 * M * N * r


def fwd_bwd_flops(M, N, K, r):
    return 4 * M * N * K + 6 * M * r * (N + K)


def nf4_bytes(N, K, bs=64, dq=256):
    n = N * K
    nb = -(-n // bs)
    return -(-n // 2) + nb + 4 * (-(-nb // dq)) + 4


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    sm_max_mhz=float(d.get("sm_max_mhz", 1965.0)), source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, sm_max_mhz=1965.0,
                source="fallback")


def bf16_peak(peaks, clocks):
    """The dense bf16 denominator of every tensor-bound fraction: the burst
    figure (cuBLAS bf16 GEMM timed alone at full clock), whatever the clock
    did.  When the power cap held the SM clock below its maximum during the
    timed region (a seconds-long step), the lines also give the fraction of
    the sustained figure and of the burst figure scaled to the median clock.
    Returns (peak TFLOP/s, description)."""
    mhz, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz") or peaks["sm_max_mhz"]
    capped = "sw_power_cap" in (clocks.get("reasons") or [])
    note = (f"SM clock median {mhz:.0f} of {mx:.0f} MHz in the timed region"
            + (", sw_power_cap active" if capped else "")) if mhz is not None else "clock unknown"
    return peaks["bf16"], f"{peaks['source']} burst bf16 ({note})"


def clock_scaled_peak(peaks, clocks):
    """The burst figure scaled by median / maximum SM clock of the run."""
    mhz, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz") or peaks["sm_max_mhz"]
    if not mhz:
        return peaks["bf16"]
    return peaks["bf16"] * min(1.0, mhz / mx)


# dram__bytes_read.sum + dram__bytes_write.sum per launch of the dominant
# kernel, from one ncu capture, keyed by the SHA-256 (first 16 hex digits) of
# the sources that define the kernel at capture time.  When those sources
# change the figure no longer describes the kernel and the line reports null.
TRAFFIC = {
    # per launch, averaged over one layer's 7 linears (4 x 8192^2, 2 x 22016 x 8192,
    # 8192 x 22016) at 2048 tokens, one capture of each shape
    ("fused_dgrad", "stack_65b"): {"sha": "9be4da7b80466d50", "bytes_per_launch": 171768722},
    ("fused_fwd", "stack_65b"): {"sha": "9be4da7b80466d50", "bytes_per_launch": 157108553},
}
KERNEL_SOURCES = {
    "fused_fwd": ("gemm_tc2.cu", "tc_common.cuh", "tc_ptx.cuh"),
    "fused_dgrad": ("gemm_tc2.cu", "tc_common.cuh", "tc_ptx.cuh"),
}


def sources_sha(kernel):
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, ()):
        with open(os.path.join(ROOT, "bit_nf4_quantized_17_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_of(kernel, workload):
    t = TRAFFIC.get((kernel, workload))
    if t is None or t["sha"] != sources_sha(kernel):
        return None
    return t["bytes_per_launch"]


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    """nvidia-smi samples (200 ms) taken while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self._summary = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self._summary is not None:
            return self._summary
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
                except ValueError:
                    continue
            os.unlink(self.path)
        if rows:
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            reasons = sorted({names[i] for *_, r in rows for i, v in enumerate(r)
                              if v == "Active"})
            out = {"sm_mhz": statistics.median(c for c, *_ in rows),
                   "sm_max_mhz": max(m for _, m, *_ in rows),
                   "power_w_max": max(p for _, _, p, _ in rows), "samples": len(rows),
                   "reasons": reasons}
        self._summary = out
        return out


def _lib():
    from bit_nf4_quantized_17_b200 import dp
    from bit_nf4_quantized_17_b200 import qlora as Q
    from bit_nf4_quantized_17_b200 import workloads as WL
    return dp, Q, WL


def kernel_lines(kt, work, peaks, bf16, bf16_kind, clocks=None):
    """Per-kernel achieved rate from the library's per-launch CUDA events.

    ``work`` maps a name to (kernel kind, "hbm" | "tensor", algorithmic bytes
    or FLOPs of all its launches in one step, launches per step); the
    average launch then processes work / launches, and achieved = that
    per-launch work / the average event time of the kind's launches."""
    out = {}
    for name, (kind, bound, per_step, launches_per_step) in work.items():
        total_ms, n = kt[kind]
        if n == 0 or launches_per_step == 0:
            continue
        avg_s = total_ms * 1e-3 / n
        per_launch = per_step / launches_per_step
        if bound == "hbm":
            achieved, peak, unit = per_launch / avg_s / 1e9, peaks["hbm"], "GB/s"
            kind_s = f"{peaks['source']} HBM copy bandwidth"
        else:
            achieved, peak, unit = per_launch / avg_s / 1e12, bf16, "TFLOP/s"
            kind_s = bf16_kind
        line = {"bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
                "frac": round(achieved / peak, 4), "avg_us": round(avg_s * 1e6, 2),
                "launches": n, "total_ms": round(total_ms, 4),
                "algorithmic_per_launch": per_launch, "peak_kind": kind_s}
        if bound == "tensor":
            line["frac_of_sustained"] = round(achieved / peaks["bf16_sustained"], 4)
            if clocks is not None:
                line["frac_of_clock_scaled_burst"] = round(
                    achieved / clock_scaled_peak(peaks, clocks), 4)
        out[name] = line
    return out


def roofline_of(kernels, workload):
    name = max(kernels, key=lambda k: kernels[k]["total_ms"])
    d = kernels[name]
    return {"bound": d["bound"], "achieved": d["achieved"], "peak": d["peak"], "unit": d["unit"],
            "frac": d["frac"], "traffic": traffic_of(name, workload), "kernel": name,
            "avg_launch_us": d["avg_us"], "algorithmic_per_launch": d["algorithmic_per_launch"],
            "peak_kind": d["peak_kind"]}


# ------------------------------------------------------------- the stack --

class Stack:
    """A decoder stack of quantised linears resident on one GPU.

    Per linear: the NF4 arrays (quantised once here), A and B (bf16) and the
    saved U = X A^T (fp32).  Per linear position j of a layer and per slot:
    the activations X_j, dY_j and the outputs Y_j, dX_j, shared by the
    layers (each layer overwrites Y_j and dX_j).  Per layer and slot: one
    flat fp32 buffer of its 7 linears' dA and dB.  Two slots let the
    end-to-end run upload one step's inputs and download the previous step's
    results while a step computes."""

    def __init__(self, name, layers, M, dev, rank, slots=1):
        dp, Q, WL = _lib()
        self.Q, self.dp = Q, dp
        wl = WL.WORKLOADS[name]
        self.name, self.layers, self.M = name, layers, M
        self.shapes = wl.linears
        self.per_layer_flops = sum(fwd_bwd_flops(M, s.d_out, s.d_in, s.r) for s in self.shapes)
        self.flops = self.per_layer_flops * layers
        qws = torch.zeros(max(Q.qlora_nf4_sizes(s.d_out, s.d_in)["workspace"]
                              for s in self.shapes), dtype=torch.uint8, device=dev)
        self.lin = []
        self.resident_nf4_bytes = 0
        for l in range(layers):
            row = []
            for j, sh in enumerate(self.shapes):
                seed = WL.stack_seed(l, j)
                W = WL.weight(sh, seed, dev)
                q = Q.QuantizedWeight.empty(sh.d_out, sh.d_in, 64, 256, Q.QLORA_TABLE_NF4, dev)
                Q.qlora_quantize(W, out=q, workspace=qws, check=False)
                del W
                self.resident_nf4_bytes += q.nbytes
                row.append({"q": q, "A": WL.lora_a(sh, seed, dev), "B": WL.lora_b(sh, seed, dev),
                            "U": torch.empty((M, sh.r), dtype=torch.float32, device=dev)})
            self.lin.append(row)
        torch.cuda.synchronize()
        Q.qlora_check(qws)
        del qws
        # one forward and one backward workspace per distinct shape: the calls
        # are ordered on one stream, so linears of a shape share them
        self.ws = {}
        for sh in self.shapes:
            key = (sh.d_out, sh.d_in, sh.r)
            if key not in self.ws:
                fb, bb = Q.qlora_linear_workspace(M, *key)
                self.ws[key] = (torch.zeros(fb, dtype=torch.uint8, device=dev),
                                torch.zeros(bb, dtype=torch.uint8, device=dev))
        self.acts = []
        self.grads = []
        for sl in range(slots):
            a = []
            for j, sh in enumerate(self.shapes):
                tok = WL.stack_seed(0, j) + 1000 * (rank + 1) + 7919 * sl
                a.append({"X": WL.activations(sh, M, tok, dev), "dY": WL.grad_output(sh, M, tok, dev),
                          "Y": torch.empty((M, sh.d_out), dtype=torch.bfloat16, device=dev),
                          "dX": torch.empty((M, sh.d_in), dtype=torch.bfloat16, device=dev)})
            self.acts.append(a)
            self.grads.append([dp.LayerBucket([(s.r, s.d_in, s.d_out) for s in self.shapes], dev)
                               for _ in range(layers)])
        torch.cuda.synchronize()

    def kernel_work(self):
        """Algorithmic FLOPs per step of the timed kernel kinds, and launches."""
        Q = self.Q
        M, L = self.M, self.layers
        fwd = sum(2 * M * s.d_out * s.d_in + 2 * M * s.d_out * s.r for s in self.shapes) * L
        dgrad = sum(2 * M * s.d_out * s.d_in + 2 * M * s.d_in * s.r for s in self.shapes) * L
        lora = sum(4 * M * s.d_in * s.r + 4 * M * s.d_out * s.r for s in self.shapes) * L
        n = len(self.shapes) * L
        return {"fused_fwd": (Q.QLORA_KERNEL_FUSED_FWD, "tensor", fwd, n),
                "fused_dgrad": (Q.QLORA_KERNEL_FUSED_DGRAD, "tensor", dgrad, n),
                "lora_gemms": (Q.QLORA_KERNEL_LORA_GEMM, "tensor", lora, 4 * n)}

    def step(self, slot=0, world=1, ev=None):
        """Forward of every linear in layer order, then the backward in reverse
        order; with world > 1 each layer's gradient buffer is all-reduced as
        soon as its backward is enqueued."""
        Q = self.Q
        acts, grads = self.acts[slot], self.grads[slot]
        if ev is not None:
            ev[0].record()
        for row in self.lin:
            for j, (p, sh) in enumerate(zip(row, self.shapes)):
                a = acts[j]
                Q.qlora_linear_fwd(p["q"], p["A"], p["B"], sh.alpha, a["X"], Y=a["Y"],
                                   U_save=p["U"], workspace=self.ws[(sh.d_out, sh.d_in, sh.r)][0])
        if ev is not None:
            ev[1].record()
        works = []
        for l in reversed(range(self.layers)):
            row = self.lin[l]
            for j in reversed(range(len(self.shapes))):
                p, sh, a = row[j], self.shapes[j], acts[j]
                dA, dB = grads[l].views[j]
                Q.qlora_linear_bwd(p["q"], p["A"], p["B"], sh.alpha, a["X"], p["U"], a["dY"],
                                   dX=a["dX"], dA=dA, dB=dB,
                                   workspace=self.ws[(sh.d_out, sh.d_in, sh.r)][1])
            if world > 1:
                works.append(grads[l].allreduce(async_op=True))
        for w in works:
            if w is not None:
                w.wait()
        if ev is not None:
            ev[2].record()

    def check(self):
        for fws, bws in self.ws.values():
            self.Q.qlora_check(fws)
            self.Q.qlora_check(bws)


def time_stack(st, steps, warmup, world, local, peaks, kinds_pass2=True):
    """Warm-up, then `steps` timed steps between CUDA events on the compute
    stream (barrier + synchronise on both sides), with no events between the
    library's launches; then the same steps again with the library's launch
    events on, for the fused kernels' times, and once more for the rank-r
    GEMMs'.  Returns the measurement dict."""
    dp, Q, _ = _lib()
    dev = torch.device("cuda", local)
    for i in range(warmup):
        st.step(0, world)
    torch.cuda.synchronize()
    st.check()
    barrier(world)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_lin = len(st.shapes) * st.layers
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        launches0 = Q.qlora_launch_count()
        start.record()
        for i in range(steps):
            st.step(0, world, ev=evs[i])
        end.record()
        launches = Q.qlora_launch_count() - launches0
        torch.cuda.synchronize()
        barrier(world)
    clocks = clk.summary()
    # per-kernel times in separate passes: a launch event between the rank-r
    # kernel and the fused kernel would also stop their programmatic overlap
    Q.qlora_timing_begin((Q.QLORA_KERNEL_FUSED_FWD, Q.QLORA_KERNEL_FUSED_DGRAD),
                         max_launches=min(65536, 2 * n_lin * steps + 16))
    for i in range(steps):
        st.step(0, world)
    torch.cuda.synchronize()
    kt = Q.qlora_timing_end()
    if kinds_pass2:
        Q.qlora_timing_begin((Q.QLORA_KERNEL_LORA_GEMM,),
                             max_launches=min(65536, 4 * n_lin * steps + 16))
        for i in range(steps):
            st.step(0, world)
        torch.cuda.synchronize()
        kt[Q.QLORA_KERNEL_LORA_GEMM] = Q.qlora_timing_end()[Q.QLORA_KERNEL_LORA_GEMM]
    st.check()
    ms = dp.max_over_ranks(start.elapsed_time(end), dev) / steps
    t_fwd = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    t_bwd = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    bf16, bf16_kind = bf16_peak(peaks, clocks)
    kernels = kernel_lines(kt, st.kernel_work(), peaks, bf16, bf16_kind, clocks)
    fused_ms = sum(kernels[k]["total_ms"] for k in ("fused_fwd", "fused_dgrad") if k in kernels)
    return {"ms_per_step": ms, "launches": launches, "clocks": clocks, "kernels": kernels,
            "fwd_ms": t_fwd, "bwd_ms": t_bwd, "bf16": bf16, "bf16_kind": bf16_kind,
            "fused_share": fused_ms / steps / ms}


def e2e_stack(st, steps, warmup, world, local):
    """The same step through the C ABI with host buffers: every step copies
    its activations (X_j, dY_j of the 7 positions) in from pinned host memory
    and its results (dX_j of the 7 positions and every layer's dA, dB) out to
    pinned host memory.  Copies run on their own streams (one per direction)
    and two device slots alternate, so that the next step's upload and the
    previous step's download overlap this step's compute."""
    dp, Q, _ = _lib()
    dev = torch.device("cuda", local)
    host_in = [[{k: a[k].cpu().pin_memory() for k in ("X", "dY")} for a in st.acts[s]]
               for s in range(2)]
    host_dx = [[torch.empty_like(a["dX"], device="cpu").pin_memory() for a in st.acts[s]]
               for s in range(2)]
    host_g = [[torch.empty_like(g.flat, device="cpu").pin_memory() for g in st.grads[s]]
              for s in range(2)]
    h2d = sum(t.numel() * t.element_size() for d in host_in[0] for t in d.values())
    d2h = (sum(t.numel() * t.element_size() for t in host_dx[0]) +
           sum(t.numel() * t.element_size() for t in host_g[0]))
    compute = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def run(n):
        up.wait_stream(compute)
        done_c, done_d = [], []
        for i in range(n):
            j = i % 2
            with torch.cuda.stream(up):
                if i >= 2:  # the slot's previous step has computed and downloaded
                    up.wait_event(done_c[i - 2])
                    up.wait_event(done_d[i - 2])
                for a, h in zip(st.acts[j], host_in[j]):
                    a["X"].copy_(h["X"], non_blocking=True)
                    a["dY"].copy_(h["dY"], non_blocking=True)
                uploaded = torch.cuda.Event()
                uploaded.record(up)
            compute.wait_event(uploaded)
            st.step(j, world)
            ev = torch.cuda.Event()
            ev.record(compute)
            done_c.append(ev)
            with torch.cuda.stream(down):
                down.wait_event(ev)
                for a, h in zip(st.acts[j], host_dx[j]):
                    h.copy_(a["dX"], non_blocking=True)
                for g, h in zip(st.grads[j], host_g[j]):
                    h.copy_(g.flat, non_blocking=True)
                ev2 = torch.cuda.Event()
                ev2.record(down)
                done_d.append(ev2)
        compute.wait_stream(up)
        compute.wait_stream(down)

    run(warmup)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(compute)
    run(steps)
    e1.record(compute)
    torch.cuda.synchronize()
    ms = dp.max_over_ranks(e0.elapsed_time(e1), dev) / steps
    return {"value": round(st.flops * world / (ms * 1e-3) / 1e12, 3), "unit": UNIT,
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "path": "pinned host -> device copies of the step's activations (upload stream), "
                    "qlora_linear_fwd / qlora_linear_bwd of every linear through the C ABI, "
                    "device -> pinned host copies of dX and every layer's dA, dB (download "
                    "stream); two device slots, so that copies of neighbouring steps overlap "
                    "the compute"}


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def stack_config(name, layers, world):
    desc = {
        "stack_65b": "65B-shaped stack: {L} layers x 7 linears (q,k,v,o 8192x8192; gate,up "
                     "22016x8192; down 8192x22016), W ~ N(0,0.015^2) quantised once to NF4 b64 + "
                     "double quant b256 and resident, LoRA r=64 alpha=16 on every linear, "
                     "M=2048 (4x512) tokens per GPU",
        "stack_7b": "7B-shaped stack: {L} layers x 7 linears (q,k,v,o 4096x4096; gate,up "
                    "11008x4096; down 4096x11008), W ~ N(0,0.02^2) quantised once to NF4 b64 + "
                    "double quant b256 and resident, LoRA r=16 alpha=32 on every linear, "
                    "M=2048 (1x2048) tokens per GPU",
    }[name].format(L=layers)
    return {
        "workload": f"{name}: {desc}; step = forward of every linear in layer order + backward "
                    "(dX, dA, dB) in reverse order",
        "global_batch": (4 if name == "stack_65b" else 1) * world,
        "seq_len": 512 if name == "stack_65b" else 2048,
        "parallelism": f"dp{world}",
        "layers": layers,
        "l2": "weights stream from HBM: the resident stack is far larger than the 126 MB L2",
    }


# ------------------------------------------------- single-linear workloads --

class InputSet:
    def __init__(self, shape, M, seed, rank, dev):
        dp, Q, WL = _lib()
        self.W = WL.weight(shape, seed, dev)
        self.A = WL.lora_a(shape, seed, dev)
        self.B = WL.lora_b(shape, seed, dev)
        tok_seed = seed + 1000 * (rank + 1)
        self.X = WL.activations(shape, M, tok_seed, dev)
        self.dY = WL.grad_output(shape, M, tok_seed, dev)
        N, K, r = shape.d_out, shape.d_in, shape.r
        self.q = Q.QuantizedWeight.empty(N, K, 64, 256, Q.QLORA_TABLE_NF4, dev)
        self.qws = torch.zeros(Q.qlora_nf4_sizes(N, K)["workspace"], dtype=torch.uint8, device=dev)
        fwd_b, bwd_b = Q.qlora_linear_workspace(M, N, K, r)
        self.fws = torch.zeros(fwd_b, dtype=torch.uint8, device=dev)
        self.bws = torch.zeros(bwd_b, dtype=torch.uint8, device=dev)
        self.Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        self.U = torch.empty((M, r), dtype=torch.float32, device=dev)
        self.dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        self.grads = dp.GradBucket(r, K, N, dev)
        self.dA, self.dB = self.grads.dA, self.grads.dB


SINGLE = {  # name: (workload, linear indices, tokens, input sets, quantise inside the step, description)
    "attn_4096": ("attn_4096", [0], 4096, 3, False,
                  "7B attention projection, W 4096x4096 bf16 N(0,0.02^2) + 0.1% outliers at 8 "
                  "sigma, NF4 b64 + double quant b256, LoRA r=16 alpha=32, M=4096 (8x512); step "
                  "= fwd + bwd (W quantised before timing, offline as on the pages)"),
    "attn_4096_with_quantise": ("attn_4096", [0], 4096, 3, True,
                                "the same with qlora_quantize of W inside every step"),
    "mlp_8192": ("mlp_11008", [0, 1], 8192, 2, False,
                 "7B MLP gate/up 4096->11008 and down 11008->4096, r=64 alpha=16, M=8192; step = "
                 "fwd of both linears + bwd in reverse (W quantised before timing)"),
    "single_256": ("single_256", [0], 16, 3, True,
                   "single linear 256x256 fp32 W, r=8 alpha=16, M=16; step = quantise + fwd + bwd"),
}


def time_single(name, steps, warmup, peaks, dev):
    """One of the single-linear workloads, its steps captured as one CUDA graph
    (the host's launch gaps taken out); three input sets > L2 rotate."""
    dp, Q, WL = _lib()
    wl_name, idx, M, n_sets, quant, desc = SINGLE[name]
    shapes = [WL.WORKLOADS[wl_name].linears[j] for j in idx]
    sets = [[InputSet(sh, M, WL.stack_seed(0, j) + 100 * i, 0, dev) for sh, j in zip(shapes, idx)]
            for i in range(n_sets)]
    for g in sets:
        for s in g:
            Q.qlora_quantize(s.W, out=s.q, workspace=s.qws, check=False)
    flops = sum(fwd_bwd_flops(M, sh.d_out, sh.d_in, sh.r) for sh in shapes)

    def step(group):
        if quant:
            for s in group:
                Q.qlora_quantize(s.W, out=s.q, workspace=s.qws, check=False)
        for s, sh in zip(group, shapes):
            Q.qlora_linear_fwd(s.q, s.A, s.B, sh.alpha, s.X, Y=s.Y, U_save=s.U, workspace=s.fws)
        for s, sh in reversed(list(zip(group, shapes))):
            Q.qlora_linear_bwd(s.q, s.A, s.B, sh.alpha, s.X, s.U, s.dY, dX=s.dX, dA=s.dA,
                               dB=s.dB, workspace=s.bws)

    for i in range(warmup):
        step(sets[i % n_sets])
    torch.cuda.synchronize()
    def capture():
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cap):
            with torch.cuda.graph(graph, stream=cap):
                for i in range(steps):
                    step(sets[i % n_sets])
        torch.cuda.current_stream().wait_stream(cap)
        torch.cuda.synchronize()
        return graph

    # the timed graph holds the library's launches only (no launch events)
    l0 = Q.qlora_launch_count()
    graph = capture()
    launches = Q.qlora_launch_count() - l0
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index or 0) as clk:
        torch.cuda.synchronize()
        start.record()
        graph.replay()
        end.record()
        torch.cuda.synchronize()
    del graph
    # the fused kernels' and the quantiser's times from a second graph of the
    # same steps, with the library's launch events captured into it (an event
    # before a fused kernel makes it start after its U or V launch ends, where
    # the timed graph lets the two overlap)
    kinds = (Q.QLORA_KERNEL_FUSED_FWD, Q.QLORA_KERNEL_FUSED_DGRAD, Q.QLORA_KERNEL_QUANTIZE)
    Q.qlora_timing_begin(kinds, max_launches=6 * len(shapes) * steps + 16)
    graph = capture()
    graph.replay()
    torch.cuda.synchronize()
    del graph  # it refers to the library's timing events
    kt = Q.qlora_timing_end()
    # the rank-r products from eager launches of the same steps
    Q.qlora_timing_begin((Q.QLORA_KERNEL_LORA_GEMM,), max_launches=8 * len(shapes) * steps + 16)
    for i in range(steps):
        step(sets[i % n_sets])
    torch.cuda.synchronize()
    kt2 = Q.qlora_timing_end()
    kt[Q.QLORA_KERNEL_LORA_GEMM] = kt2[Q.QLORA_KERNEL_LORA_GEMM]
    for g in sets:
        for s in g:
            Q.qlora_check(s.fws)
            Q.qlora_check(s.bws)
    ms = start.elapsed_time(end) / steps
    clocks = clk.summary()
    bf16, bf16_kind = bf16_peak(peaks, clocks)
    work = {
        "fused_fwd": (Q.QLORA_KERNEL_FUSED_FWD, "tensor",
                      sum(2 * M * s.d_out * s.d_in + 2 * M * s.d_out * s.r for s in shapes),
                      len(shapes)),
        "fused_dgrad": (Q.QLORA_KERNEL_FUSED_DGRAD, "tensor",
                        sum(2 * M * s.d_out * s.d_in + 2 * M * s.d_in * s.r for s in shapes),
                        len(shapes)),
        "lora_gemms": (Q.QLORA_KERNEL_LORA_GEMM, "tensor",
                       sum(4 * M * s.d_in * s.r + 4 * M * s.d_out * s.r for s in shapes),
                       4 * len(shapes)),
    }
    if quant:
        work["quantize_blocks"] = (Q.QLORA_KERNEL_QUANTIZE, "hbm",
                                   sum(2 * s.d_out * s.d_in + s.d_out * s.d_in // 2 +
                                       4 * (s.d_out * s.d_in // 64) for s in shapes), len(shapes))
    if M <= 16:  # decode-sized: the rank-r kernels are not the tensor-core GEMMs
        work.pop("lora_gemms")
    kernels = kernel_lines(kt, work, peaks, bf16, bf16_kind, clocks)
    value = flops / (ms * 1e-3) / 1e12
    nf4 = sum(nf4_bytes(s.d_out, s.d_in) for s in shapes)
    return {"workload": f"{name}: {desc}", "value": round(value, 3), "unit": UNIT,
            "ms_per_step": round(ms, 4), "frac_of_bf16_peak": round(value / bf16, 4),
            "peak": bf16, "peak_kind": bf16_kind,
            "nf4_weight_gbs": round(2 * nf4 / (ms * 1e-3) / 1e9, 1), "gpu_launches": launches,
            "launch": "one CUDA graph of the timed steps", "steps": steps,
            "l2": f"{n_sets} rotating input sets", "kernels": kernels, "clocks": clocks}


def time_decode(peaks, dev, steps=50, warmup=5):
    """Decode-shaped gate/up linear (11008 x 4096, r = 64) at M = 1 and 16:
    forward + backward, 8 rotating weight copies (8 x 23 MB > L2)."""
    dp, Q, WL = _lib()
    shape = WL.WORKLOADS["mlp_11008"].linears[0]
    N, K, r = shape.d_out, shape.d_in, shape.r
    copies = []
    for c in range(8):
        W = WL.weight(shape, 7 * c, dev)
        copies.append(Q.qlora_quantize(W))
        del W
    A, B = WL.lora_a(shape, 0, dev), WL.lora_b(shape, 0, dev)
    out = {}
    for M in (1, 16):
        X, dY = WL.activations(shape, M, 3, dev), WL.grad_output(shape, M, 3, dev)
        fb, bb = Q.qlora_linear_workspace(M, N, K, r)
        fws = torch.zeros(fb, dtype=torch.uint8, device=dev)
        bws = torch.zeros(bb, dtype=torch.uint8, device=dev)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        U = torch.empty((M, r), dtype=torch.float32, device=dev)
        dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        dA = torch.empty((r, K), dtype=torch.float32, device=dev)
        dB = torch.empty((N, r), dtype=torch.float32, device=dev)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for i in range(warmup + steps):
            if i == warmup:
                torch.cuda.synchronize()
                Q.qlora_timing_begin((Q.QLORA_KERNEL_FUSED_FWD, Q.QLORA_KERNEL_FUSED_DGRAD),
                                     max_launches=4 * steps)
            q = copies[i % 8]
            e = evs[i - warmup] if i >= warmup else None
            if e:
                e[0].record()
            Q.qlora_linear_fwd(q, A, B, shape.alpha, X, Y=Y, U_save=U, workspace=fws)
            if e:
                e[1].record()
            Q.qlora_linear_bwd(q, A, B, shape.alpha, X, U, dY, dX=dX, dA=dA, dB=dB, workspace=bws)
            if e:
                e[2].record()
        torch.cuda.synchronize()
        kt = Q.qlora_timing_end()
        t_f = statistics.median(e[0].elapsed_time(e[1]) for e in evs) * 1e-3
        t_b = statistics.median(e[1].elapsed_time(e[2]) for e in evs) * 1e-3
        # the same calls replayed from CUDA graphs (one forward and one
        # backward graph per weight copy), as a decode loop would run them:
        # the host's per-call cost leaves the measurement
        graphs = []
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cap):
            for c in range(8):
                gf, gb = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
                with torch.cuda.graph(gf, stream=cap):
                    Q.qlora_linear_fwd(copies[c], A, B, shape.alpha, X, Y=Y, U_save=U, workspace=fws)
                with torch.cuda.graph(gb, stream=cap):
                    Q.qlora_linear_bwd(copies[c], A, B, shape.alpha, X, U, dY, dX=dX, dA=dA, dB=dB,
                                       workspace=bws)
                graphs.append((gf, gb))
        torch.cuda.current_stream().wait_stream(cap)
        torch.cuda.synchronize()
        gevs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for i in range(warmup + steps):
            gf, gb = graphs[i % 8]
            e = gevs[i - warmup] if i >= warmup else None
            if e:
                e[0].record()
            gf.replay()
            if e:
                e[1].record()
            gb.replay()
            if e:
                e[2].record()
        torch.cuda.synchronize()
        g_f = statistics.median(e[0].elapsed_time(e[1]) for e in gevs) * 1e-3
        g_b = statistics.median(e[1].elapsed_time(e[2]) for e in gevs) * 1e-3
        del graphs
        Q.qlora_check(fws)
        Q.qlora_check(bws)
        wb = nf4_bytes(N, K)
        # the fused kernels alone: NF4 bytes + activations in/out + adapter
        # (algorithmic HBM bytes of one launch) / average launch time
        fused = {}
        for name, kind, extra in (("fused_fwd", Q.QLORA_KERNEL_FUSED_FWD,
                                   2 * M * K + 2 * M * N + 2 * N * r),
                                  ("fused_dgrad", Q.QLORA_KERNEL_FUSED_DGRAD,
                                   2 * M * N + 2 * M * K + 2 * K * r)):
            ms, n = kt[kind]
            if n:
                avg = ms * 1e-3 / n
                alu_peak = alu_peak_ops(peaks)
                fused[name] = {"avg_us": round(avg * 1e6, 2),
                               "gbs": round((wb + extra) / avg / 1e9, 1),
                               "frac_hbm": round((wb + extra) / avg / 1e9 / peaks["hbm"], 4),
                               "nf4_frac_hbm": round(wb / avg / 1e9 / peaks["hbm"], 4),
                               "alu": {"bound": "alu",
                                       "achieved": round(EXPAND_OPS_PER_WEIGHT * N * K / avg / 1e12, 2),
                                       "peak": round(alu_peak / 1e12, 2), "unit": "T lane-ops/s",
                                       "frac": round(EXPAND_OPS_PER_WEIGHT * N * K / avg / alu_peak, 4),
                                       "ops_per_weight": EXPAND_OPS_PER_WEIGHT}}
        out[f"M{M}"] = {
            "fwd_us": round(t_f * 1e6, 2), "bwd_us": round(t_b * 1e6, 2),
            "fwd_nf4_gbs": round(wb / t_f / 1e9, 1), "bwd_nf4_gbs": round(wb / t_b / 1e9, 1),
            "fwd_frac_hbm": round(wb / t_f / 1e9 / peaks["hbm"], 4),
            "bwd_frac_hbm": round(wb / t_b / 1e9 / peaks["hbm"], 4),
            "graph_fwd_us": round(g_f * 1e6, 2), "graph_bwd_us": round(g_b * 1e6, 2),
            "graph_fwd_frac_hbm": round(wb / g_f / 1e9 / peaks["hbm"], 4),
            "graph_bwd_frac_hbm": round(wb / g_b / 1e9 / peaks["hbm"], 4),
            "kernels": fused,
        }
    out["workload"] = "mlp gate/up 11008x4096, r=64, alpha=16; NF4 bytes per pass " \
                      f"{nf4_bytes(N, K)}; 8 rotating weight copies; median of {steps}"
    return out


# Minimum ALU work of the exact compute weight per weight: 21 byte-permute,
# shift and logic operations per 8 weights for the lookup, and 16 per 64 weights
# for the block's tables (the conversions and the table permutes)
EXPAND_OPS_PER_WEIGHT = 21 / 8 + 16 / 64


def alu_peak_ops(peaks):
    """ALU lane-operations per second: 64 lanes per clock on each of the
    device's SMs at the maximum SM clock."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count if torch.cuda.is_available() else 148
    return sms * 64 * peaks.get("sm_max_mhz", 1965.0) * 1e6


def time_merge(peaks, dev, steps=20):
    """qlora_merge of the 7B attention projection's quantised weight into bf16
    (the deployment step after training): NF4 bytes + A + B read, 2 bytes per
    weight written; three weight copies rotate."""
    dp, Q, WL = _lib()
    shape = WL.WORKLOADS["attn_4096"].linears[0]
    N, K, r = shape.d_out, shape.d_in, shape.r
    qs = [Q.qlora_quantize(WL.weight(shape, 100 * i, dev)) for i in range(3)]
    A, B = WL.lora_a(shape, 0, dev), WL.lora_b(shape, 0, dev)
    outs = [torch.empty((N, K), dtype=torch.bfloat16, device=dev) for _ in range(3)]
    for i in range(3):
        Q.qlora_merge(qs[i], A, B, shape.alpha, out=outs[i])
    torch.cuda.synchronize()
    Q.qlora_timing_begin((Q.QLORA_KERNEL_MERGE,), max_launches=steps)
    for i in range(steps):
        Q.qlora_merge(qs[i % 3], A, B, shape.alpha, out=outs[i % 3])
    torch.cuda.synchronize()
    ms, n = Q.qlora_timing_end()[Q.QLORA_KERNEL_MERGE]
    t = ms * 1e-3 / max(n, 1)
    nbytes = nf4_bytes(N, K) + 2 * r * (N + K) + 2 * N * K
    return {"us": round(t * 1e6, 2), "gbs": round(nbytes / t / 1e9, 1),
            "frac_hbm": round(nbytes / t / 1e9 / peaks["hbm"], 4),
            "workload": f"{N}x{K} r={r}: NF4 + A + B read, bf16 W written; {n} launches"}


# ------------------------------------------------------- the CPU oracle ----

def _cpu_info():
    from threadpoolctl import threadpool_info
    cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    model = ""
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return cores, model


_ORACLE_INPUTS = {}


def _oracle_inputs(shape, tokens, seed):
    """Seeded inputs of one linear as numpy arrays and the oracle's encoding
    of W (cached: the stacks' samples reuse them from step to step)."""
    import oracle
    dp, Q, WL = _lib()
    key = (shape, tokens, seed)
    if key not in _ORACLE_INPUTS:
        inp = WL.linear_inputs(shape, tokens, seed)
        f = lambda t: t.float().numpy()
        W = f(inp["W"])
        _ORACLE_INPUTS[key] = (W, oracle.quantize(W, 64, 256), f(inp["A"]), f(inp["B"]),
                               f(inp["X"]), f(inp["dY"]))
    return _ORACLE_INPUTS[key]


def oracle_linear_times(shape, tokens, seed=0, repeats=1):
    """The oracle on one linear: (seconds to restore the compute weight from
    the quantised W, seconds of fwd + bwd on `tokens` tokens), medians of
    `repeats`.  Quantisation itself is offline on both arms of the stacks."""
    import oracle
    W, qt, A, B, X, dY = _oracle_inputs(shape, tokens, seed)
    t_deq, t_mm = [], []
    for _ in range(repeats):
        t0 = time.perf_counter()
        w_bf16 = oracle.compute_weight(qt).reshape(W.shape)
        t1 = time.perf_counter()
        oracle.linear_fwd(w_bf16, A, B, shape.alpha, X)
        oracle.linear_bwd(w_bf16, A, B, shape.alpha, X, dY)
        t2 = time.perf_counter()
        t_deq.append(t1 - t0)
        t_mm.append(t2 - t1)
    return statistics.median(t_deq), statistics.median(t_mm)


def cpu_stack_estimate(name, layers, M, sample_tokens=CPU_SAMPLE_TOKENS, repeats=1):
    """The oracle timed on one linear of the stack (the first of the layer)
    and extrapolated to the whole step: the restore of the compute weight
    scales with N K, the products with M N K (plus the rank-r terms)."""
    dp, Q, WL = _lib()
    shapes = WL.WORKLOADS[name].linears
    s0 = shapes[0]
    t_deq, t_mm = oracle_linear_times(s0, sample_tokens, 0, repeats)
    per_w = t_deq / (s0.d_out * s0.d_in)
    per_f = t_mm / fwd_bwd_flops(sample_tokens, s0.d_out, s0.d_in, s0.r)
    t_step = layers * sum(per_w * s.d_out * s.d_in + per_f * fwd_bwd_flops(M, s.d_out, s.d_in, s.r)
                          for s in shapes)
    flops = layers * sum(fwd_bwd_flops(M, s.d_out, s.d_in, s.r) for s in shapes)
    cores, model = _cpu_info()
    return {"value": flops / t_step / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "cpu": model, "seconds_sample": round(t_deq + t_mm, 3),
            "seconds_per_step_extrapolated": round(t_step, 1),
            "sample": f"oracle restore of the compute weight of one {s0.d_out}x{s0.d_in} W + fwd/bwd "
                      f"on {sample_tokens} tokens (median of {repeats}), extrapolated to the whole "
                      f"step ({layers} layers x {len(shapes)} linears, {M} tokens) by N*K for the "
                      f"restore and by FLOPs for the products"}


def cpu_single(name, tokens_sample=None, repeats=1):
    """The oracle on a single-linear workload, timed like the GPU step
    (quantisation inside the timed part where the workload's step has it);
    the full token count unless `tokens_sample` (then FLOPs of the sample /
    its time)."""
    import oracle
    dp, Q, WL = _lib()
    wl_name, idx, M, _, quant, desc = SINGLE[name]
    m = tokens_sample or M
    total_t, total_f = 0.0, 0
    for j in idx:
        sh = WL.WORKLOADS[wl_name].linears[j]
        W, qt0, A, B, X, dY = _oracle_inputs(sh, m, 0)
        ts = []
        for _ in range(repeats):
            t0 = time.perf_counter()
            qt = oracle.quantize(W, 64, 256) if quant else qt0
            w_bf16 = oracle.compute_weight(qt).reshape(W.shape)
            oracle.linear_fwd(w_bf16, A, B, sh.alpha, X)
            oracle.linear_bwd(w_bf16, A, B, sh.alpha, X, dY)
            ts.append(time.perf_counter() - t0)
        total_t += statistics.median(ts)
        total_f += fwd_bwd_flops(m, sh.d_out, sh.d_in, sh.r)
    cores, model = _cpu_info()
    return {"value": total_f / total_t / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "cpu": model, "seconds": round(total_t, 3),
            "sample": f"{name}: oracle {'quantise + ' if quant else ''}restore + fwd/bwd on "
                      f"{m} of {M} tokens; FLOPs of those tokens / time"}


# --------------------------------------------------------------- our arm ---

def run_ours(args):
    dp, Q, WL = _lib()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    peaks = measured_peaks()
    name = args.workload
    layers = args.layers or WL.WORKLOADS[name].layers
    st = Stack(name, layers, STACK_TOKENS, dev, rank, slots=1 if args.no_e2e else 2)
    m = time_stack(st, args.steps, args.warmup, world, local, peaks)
    e2e = None if args.no_e2e else e2e_stack(st, args.steps, args.warmup, world, local)
    resident = st.resident_nf4_bytes
    flops, per_layer = st.flops, st.per_layer_flops
    nf4_step = 2 * sum(nf4_bytes(s.d_out, s.d_in) for s in st.shapes) * layers
    del st
    torch.cuda.empty_cache()

    extras = {}
    if rank == 0 and world == 1 and not args.no_extras:
        st7 = Stack("stack_7b", WL.WORKLOADS["stack_7b"].layers, STACK_TOKENS, dev, 0)
        m7 = time_stack(st7, max(args.steps, 10), args.warmup, 1, local, peaks,
                        kinds_pass2=False)
        extras["stack_7b"] = {
            "workload": stack_config("stack_7b", st7.layers, 1)["workload"],
            "value": round(st7.flops / (m7["ms_per_step"] * 1e-3) / 1e12, 3), "unit": UNIT,
            "ms_per_step": round(m7["ms_per_step"], 4),
            "frac_of_bf16_peak": round(st7.flops / (m7["ms_per_step"] * 1e-3) / 1e12 / m7["bf16"], 4),
            "peak_kind": m7["bf16_kind"], "resident_nf4_bytes": st7.resident_nf4_bytes,
            "gpu_launches": m7["launches"], "kernels": m7["kernels"], "clocks": m7["clocks"],
            "launch": "eager"}
        del st7
        torch.cuda.empty_cache()
        for nm in ("attn_4096", "attn_4096_with_quantise", "mlp_8192", "single_256"):
            extras[nm] = time_single(nm, 20, max(args.warmup, 3), peaks, dev)
            torch.cuda.empty_cache()
        extras["decode"] = time_decode(peaks, dev)
        extras["merge"] = time_merge(peaks, dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_stack_estimate(name, layers, STACK_TOKENS)
        if not args.no_extras:
            extras["cpu_baselines"] = {
                "single_256": cpu_single("single_256", repeats=3),
                "attn_4096": cpu_single("attn_4096", tokens_sample=256),
                "stack_7b": cpu_stack_estimate("stack_7b", 32, STACK_TOKENS)}

    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    ms = m["ms_per_step"]
    value = flops * world / (ms * 1e-3) / 1e12
    kernels = m["kernels"]
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,.) tensors of the workload's shapes, random-init adapters)",
        "config": stack_config(name, layers, world),
        "launch": "eager (one call per linear; the GPU queue stays ahead of the host)",
        "resident_nf4_bytes": resident,
        "flops_per_step": flops, "flops_per_layer": per_layer,
        "nf4_weight_gbs": round(nf4_step / (ms * 1e-3) / 1e9, 1),
        "fwd_ms": round(m["fwd_ms"], 3), "bwd_ms": round(m["bwd_ms"], 3),
        "frac_of_bf16_peak": round(value / world / m["bf16"], 4),
        "frac_of_bf16_sustained": round(value / world / peaks["bf16_sustained"], 4),
        "frac_of_clock_scaled_burst": round(value / world / clock_scaled_peak(peaks, m["clocks"]), 4),
        "peak_kind": m["bf16_kind"], "fused_share": round(m["fused_share"], 4),
        "roofline": roofline_of(kernels, name), "kernels": kernels, "cpu_baseline": cpu,
        "e2e": e2e, "gpu_launches": m["launches"], "clocks": m["clocks"], "peaks": peaks,
    }
    line.update(extras)
    print(json.dumps(line), flush=True)


# ------------------------------------------------------ reference arm ----

def run_reference(args):
    """The CPU oracle as the reference arm: each step is one bounded sample
    (one linear of the workload: restore of its compute weight + fwd/bwd on
    a token sample), extrapolated to the whole step of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    dp, Q, WL = _lib()
    name = args.workload
    layers = args.layers or WL.WORKLOADS[name].layers
    for _ in range(args.warmup):
        cpu_stack_estimate(name, layers, STACK_TOKENS)
    t0 = time.perf_counter()
    runs = [cpu_stack_estimate(name, layers, STACK_TOKENS) for _ in range(args.steps)]
    wall = time.perf_counter() - t0
    value = statistics.median(r["value"] for r in runs)
    est = statistics.median(r["seconds_per_step_extrapolated"] for r in runs)
    cpu = dict(runs[0])
    cpu["value"] = value
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": est * 1e3,
        "sample_seconds_per_step": round(wall / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,.) tensors of the workload's shapes, random-init adapters)",
        "config": stack_config(name, layers, world),
        "cpu_baseline": cpu,
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_cpu_configs(args):
    """The oracle on every configuration, for the baseline table: the single
    linears in full (configs 1-3), the stacks on one linear extrapolated."""
    dp, Q, WL = _lib()
    out = {"single_256": cpu_single("single_256", repeats=3),
           "attn_4096": cpu_single("attn_4096"),
           "mlp_8192": cpu_single("mlp_8192"),
           "stack_7b": cpu_stack_estimate("stack_7b", 32, STACK_TOKENS, sample_tokens=256),
           "stack_65b": cpu_stack_estimate("stack_65b", 80, STACK_TOKENS, sample_tokens=256)}
    for M in (1, 16):
        sh = WL.WORKLOADS["mlp_11008"].linears[0]
        t_deq, t_mm = oracle_linear_times(sh, M)
        out[f"decode_M{M}"] = {"seconds": round(t_deq + t_mm, 3),
                               "nf4_gbs": round(nf4_bytes(sh.d_out, sh.d_in) / (t_deq + t_mm) / 1e9, 4),
                               "sample": f"11008x4096 restore + fwd/bwd on {M} tokens"}
    print(json.dumps({"cpu_configs": out}), flush=True)


# ---------------------------------------------------------- one linear ----

def run_case(args):
    """One linear of a workload: quantise W once, then --iters forward (+
    backward) passes on the current stream; prints the wall time of the last
    one.  A driver for single-kernel profiles, not a benchmark result."""
    dp, Q, WL = _lib()
    wl = WL.WORKLOADS[args.case]
    shape = wl.linears[args.linear]
    M = args.tokens if args.tokens is not None else wl.tokens[0]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = WL.linear_inputs(shape, M, 0, dev)
    q = Q.qlora_quantize(inp["W"])
    N, K, r = shape.d_out, shape.d_in, shape.r
    fb, bb = Q.qlora_linear_workspace(M, N, K, r)
    fws = torch.zeros(fb, dtype=torch.uint8, device=dev)
    bws = torch.zeros(bb, dtype=torch.uint8, device=dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    U = torch.empty((M, r), dtype=torch.float32, device=dev)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    dA = torch.empty((r, K), dtype=torch.float32, device=dev)
    dB = torch.empty((N, r), dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    t = 0.0
    if args.merge:  # the adapter merged into a restored bf16 weight instead
        for _ in range(args.iters):
            t0 = time.perf_counter()
            Q.qlora_merge(q, inp["A"], inp["B"], shape.alpha)
            torch.cuda.synchronize()
            t = time.perf_counter() - t0
        print(f"{args.case}[{args.linear}] {N}x{K} r={r}: merge, last iteration {t * 1e6:.1f} us "
              f"(wall clock, not a benchmark)")
        return
    for _ in range(args.iters):
        t0 = time.perf_counter()
        Q.qlora_linear_fwd(q, inp["A"], inp["B"], shape.alpha, inp["X"], Y=Y, U_save=U,
                           workspace=fws)
        if not args.fwd_only:
            Q.qlora_linear_bwd(q, inp["A"], inp["B"], shape.alpha, inp["X"], U, inp["dY"],
                               dX=dX, dA=dA, dB=dB, workspace=bws)
        torch.cuda.synchronize()
        t = time.perf_counter() - t0
    Q.qlora_check(fws)
    Q.qlora_check(bws)
    print(f"{args.case}[{args.linear}] {N}x{K} r={r} M={M}: last iteration {t * 1e6:.1f} us "
          f"(wall clock, not a benchmark)")


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=WORKLOAD, choices=("stack_65b", "stack_7b"),
                    help="the stack the headline line measures")
    ap.add_argument("--layers", type=int, default=None,
                    help="layers of the stack (default: all of the workload's)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="only the headline stack (no other workloads, decode, merge)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--case", default=None, help="run one linear of this workload (profiling)")
    ap.add_argument("--linear", type=int, default=0)
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--fwd-only", action="store_true")
    ap.add_argument("--merge", action="store_true", help="with --case: run qlora_merge instead")
    ap.add_argument("--cpu-configs", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.case is None:
        ap.error("--warmup must be at least 3")
    if args.case is not None:
        run_case(args)
    elif args.cpu_configs:
        run_cpu_configs(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
