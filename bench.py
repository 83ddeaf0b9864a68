#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: the 7B attention projection, W 4096 x 4096 bf16 ~ N(0, 0.02^2)
with 0.1 % outliers at +-8 sigma, NF4 blocksize 64 + double quantisation
(256), LoRA r = 16, alpha = 32, X = 8 x 512 = 4096 tokens per GPU.  One step
is the whole path over one batch: quantise W, forward, backward (dX, dA, dB).
The metric counts the forward + backward FLOPs only (4MNK + 6Mr(N+K)), so the
quantisation inside each step makes the number conservative.

Three input sets (W, X, dY, outputs: ~170 MB each, 510 MB in all) rotate
between steps so that no step finds its inputs in the 126 MB L2.

With N > 1 (torchrun, one process per GPU) every rank holds the same frozen
W and its own tokens; the LoRA gradients dA, dB are summed over ranks with
one NCCL all-reduce per step (data parallelism; weak scaling).  Rank 0
prints one JSON line.

--impl reference times the CPU oracle (oracle/) on the host cores on a
bounded sample of the same workload.
"""

import argparse
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

WORKLOAD = "attn_4096"
TOKENS = 4096
METRIC = "QLoRA linear fwd+bwd TFLOP/s and NF4 weight GB/s at 1 B200; % of roofline"
UNIT = "TFLOP/s"
N_SETS = 3
CPU_TOKENS = 256   # tokens of the oracle's bounded sample (CPU baseline and reference arm)


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
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def workload_config(n_gpus):
    return {
        "workload": "attn_4096: 7B attention projection, W 4096x4096 bf16 N(0,0.02^2) + 0.1% "
                    "outliers at 8 sigma, NF4 b64 + double quant b256, LoRA r=16 alpha=32, "
                    "M=4096 tokens (8x512) per GPU; step = quantise + fwd + bwd (dX, dA, dB)",
        "global_batch": TOKENS * n_gpus,
        "seq_len": 512,
        "parallelism": f"dp{n_gpus}",
        "l2": f"{N_SETS} rotating input sets (~510 MB) > 126 MB L2",
    }


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
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v == "Active"})
        # samples under load: the upper half of the clock readings excludes idle gaps
        return {"sm_mhz": statistics.median(c for c, _, _ in rows),
                "sm_max_mhz": max(m for _, m, _ in rows), "samples": len(rows),
                "reasons": reasons}


# ----------------------------------------------------------- GPU arm -----

class InputSet:
    def __init__(self, shape, M, seed, rank, dev, Q, WL, dp):
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
        # dA and dB are views of one flat buffer: one all-reduce per step
        self.grads = dp.GradBucket(r, K, N, dev)
        self.dA, self.dB = self.grads.dA, self.grads.dB


def run_step(s, shape, Q, ev=None, world=1):
    Q.qlora_quantize(s.W, out=s.q, workspace=s.qws, check=False)
    if ev is not None:
        ev[0].record()
    Q.qlora_linear_fwd(s.q, s.A, s.B, shape.alpha, s.X, Y=s.Y, U_save=s.U, workspace=s.fws)
    if ev is not None:
        ev[1].record()
    Q.qlora_linear_bwd(s.q, s.A, s.B, shape.alpha, s.X, s.U, s.dY, dX=s.dX, dA=s.dA, dB=s.dB,
                       workspace=s.bws)
    if ev is not None:
        ev[2].record()
    if world > 1:
        s.grads.allreduce()


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


# dram__bytes_read.sum + dram__bytes_write.sum per launch from one ncu capture
# of the kernel as it is now (profiles/tc2_fused_attn_4096.md, same workload);
# to be cleared whenever the kernel changes.
TRAFFIC = {"fused_fwd": 46464256 + 5218304, "fused_dgrad": 43625728 + 3218432}


def kernel_rooflines(kt, M, N, K, r, peaks):
    """Per-kernel achieved rate from the library's per-launch CUDA events.

    Algorithmic work per launch (one linear, M tokens):
      quantise    HBM bytes 2NK (bf16 W) + NK/2 (codes) + 4 NK/64 (fp32 block absmax)
      fused fwd   FLOPs 2MNK + 2MNr  (base product + LoRA up-projection)
      fused dgrad FLOPs 2MNK + 2MKr  (dY W + V A)
      LoRA GEMMs  FLOPs 2MKr (U) + 2MNr (V) + 2MNr (dB) + 2MKr (dA), four launches
    """
    from bit_nf4_quantized_17_b200 import qlora as Q
    nb = -(-N * K // 64)
    spec = {
        "quantize_blocks": (Q.QLORA_KERNEL_QUANTIZE, "hbm", 2 * N * K + N * K // 2 + 4 * nb, 1),
        "fused_fwd": (Q.QLORA_KERNEL_FUSED_FWD, "tensor", 2 * M * N * K + 2 * M * N * r, 1),
        "fused_dgrad": (Q.QLORA_KERNEL_FUSED_DGRAD, "tensor", 2 * M * N * K + 2 * M * K * r, 1),
        "lora_gemms": (Q.QLORA_KERNEL_LORA_GEMM, "tensor", 4 * M * K * r + 4 * M * N * r, 4),
    }
    out = {}
    for name, (kind, bound, work, per_step) in spec.items():
        total_ms, n = kt[kind]
        if n == 0:
            continue
        avg_s = total_ms * 1e-3 / n
        per_launch = work / per_step
        if bound == "hbm":
            achieved, peak, unit = per_launch / avg_s / 1e9, peaks["hbm"], "GB/s"
            kind_s = f"{peaks['source']} HBM copy bandwidth"
        else:
            achieved, peak, unit = per_launch / avg_s / 1e12, peaks["bf16_sustained"], "TFLOP/s"
            kind_s = f"{peaks['source']} sustained bf16 (kernel timed inside a long step)"
        out[name] = {"bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
                     "frac": round(achieved / peak, 4), "avg_us": round(avg_s * 1e6, 2),
                     "launches": n, "total_ms": round(total_ms, 4),
                     "algorithmic_per_launch": per_launch, "peak_kind": kind_s}
    return out


def time_decode(Q, WL, dev, peaks, steps=50, warmup=5):
    """Decode-shaped gate/up linear (11008 x 4096, r = 64) at M = 1 and 16:
    forward + backward, 8 rotating weight copies (8 x 23 MB > L2)."""
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
        wb = nf4_bytes(N, K)
        # the fused kernels alone: NF4 bytes + activations in/out + adapter
        # (algorithmic HBM bytes of one launch) / average launch time
        fused = {}
        for name, kind, extra in (("fused_fwd", Q.QLORA_KERNEL_FUSED_FWD, 2 * M * K + 2 * M * N + 2 * N * r),
                                  ("fused_dgrad", Q.QLORA_KERNEL_FUSED_DGRAD, 2 * M * N + 2 * M * K + 2 * K * r)):
            ms, n = kt[kind]
            if n:
                avg = ms * 1e-3 / n
                fused[name] = {"avg_us": round(avg * 1e6, 2),
                               "gbs": round((wb + extra) / avg / 1e9, 1),
                               "frac_hbm": round((wb + extra) / avg / 1e9 / peaks["hbm"], 4)}
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


def time_merge(Q, sets, shape, peaks, steps=20):
    """qlora_merge of the bench's quantised weights into bf16 (the deployment
    step after training): NF4 bytes + A + B read, 2 bytes per weight written."""
    N, K, r = shape.d_out, shape.d_in, shape.r
    outs = [torch.empty((N, K), dtype=torch.bfloat16, device=s.A.device) for s in sets]
    for i in range(3):
        Q.qlora_merge(sets[i % N_SETS].q, sets[i % N_SETS].A, sets[i % N_SETS].B, shape.alpha,
                      out=outs[i % N_SETS])
    torch.cuda.synchronize()
    Q.qlora_timing_begin((Q.QLORA_KERNEL_MERGE,), max_launches=steps)
    for i in range(steps):
        s = sets[i % N_SETS]
        Q.qlora_merge(s.q, s.A, s.B, shape.alpha, out=outs[i % N_SETS])
    torch.cuda.synchronize()
    ms, n = Q.qlora_timing_end()[Q.QLORA_KERNEL_MERGE]
    t = ms * 1e-3 / max(n, 1)
    nbytes = nf4_bytes(N, K) + 2 * r * (N + K) + 2 * N * K
    return {"us": round(t * 1e6, 2), "gbs": round(nbytes / t / 1e9, 1),
            "frac_hbm": round(nbytes / t / 1e9 / peaks["hbm"], 4),
            "workload": f"{N}x{K} r={r}: NF4 + A + B read, bf16 W written; {n} launches"}


def cpu_oracle_sample(shape, tokens_sample, WL, min_seconds=10.0, max_repeats=20):
    """Oracle quantise of the full W + fwd/bwd on `tokens_sample` tokens,
    repeated until about `min_seconds` of CPU work (at least 3 repeats)."""
    import oracle
    from threadpoolctl import threadpool_info
    inp = WL.linear_inputs(shape, tokens_sample, 0)
    W = inp["W"].float().numpy()
    f = lambda t: t.float().numpy()
    A, B, X, dY = f(inp["A"]), f(inp["B"]), f(inp["X"]), f(inp["dY"])
    times = []
    while len(times) < 3 or (sum(times) < min_seconds and len(times) < max_repeats):
        t0 = time.perf_counter()
        qt = oracle.quantize(W, 64, 256)
        w_hat = oracle.dequantize(qt).reshape(W.shape)
        oracle.linear_fwd(w_hat, A, B, shape.alpha, X)
        oracle.linear_bwd(w_hat, A, B, shape.alpha, X, dY)
        times.append(time.perf_counter() - t0)
    cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    t = statistics.median(times)
    flops = fwd_bwd_flops(tokens_sample, shape.d_out, shape.d_in, shape.r)
    return {"value": flops / t / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"oracle quantise of the full 4096x4096 W + fwd/bwd on {tokens_sample} of "
                      f"the {TOKENS} tokens, median of {len(times)} ({sum(times):.1f} s of CPU "
                      f"work); FLOPs of those tokens / time",
            "seconds_per_sample": round(t, 3)}


def run_ours(args):
    from bit_nf4_quantized_17_b200 import dp
    from bit_nf4_quantized_17_b200 import qlora as Q
    from bit_nf4_quantized_17_b200 import workloads as WL

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
    shape = WL.WORKLOADS[WORKLOAD].linears[0]
    N, K, r, M = shape.d_out, shape.d_in, shape.r, TOKENS
    sets = [InputSet(shape, M, 100 * i, rank, dev, Q, WL, dp) for i in range(N_SETS)]
    torch.cuda.synchronize()

    for i in range(args.warmup):
        run_step(sets[i % N_SETS], shape, Q, world=world)
    torch.cuda.synchronize()
    barrier(world)

    # events recorded inside a CUDA graph must be external to be recorded when it runs
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]
           for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # per-kernel CUDA events, recorded by the library on the launching stream
    # around the two fused kernels (the dominant ones) inside the timed region
    fused_kinds = (Q.QLORA_KERNEL_FUSED_FWD, Q.QLORA_KERNEL_FUSED_DGRAD)
    use_graph = world == 1 and not args.eager
    graph = None
    if use_graph:
        # the K timed steps captured as one CUDA graph (launched once below):
        # the same kernels with the host's launch gaps taken out
        launches0 = Q.qlora_launch_count()
        Q.qlora_timing_begin(fused_kinds, max_launches=4 * args.steps)
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cap):
            with torch.cuda.graph(graph, stream=cap):
                for i in range(args.steps):
                    run_step(sets[i % N_SETS], shape, Q, ev=evs[i], world=world)
        torch.cuda.current_stream().wait_stream(cap)
        launches = Q.qlora_launch_count() - launches0
        torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        if use_graph:
            start.record()
            graph.replay()
            end.record()
        else:
            launches0 = Q.qlora_launch_count()
            Q.qlora_timing_begin(fused_kinds, max_launches=4 * args.steps)
            start.record()
            for i in range(args.steps):
                run_step(sets[i % N_SETS], shape, Q, ev=evs[i], world=world)
            end.record()
            launches = Q.qlora_launch_count() - launches0
        torch.cuda.synchronize()
        # the graph refers to the library's timing events: release it first
        del graph
        kt = Q.qlora_timing_end()
        barrier(world)
    # the other kernels in a second pass over the same steps (their events
    # would otherwise add a gap to every launch of the timed region)
    Q.qlora_timing_begin((Q.QLORA_KERNEL_QUANTIZE, Q.QLORA_KERNEL_LORA_GEMM),
                         max_launches=8 * args.steps)
    for i in range(args.steps):
        run_step(sets[i % N_SETS], shape, Q, world=world)
    torch.cuda.synchronize()
    kt2 = Q.qlora_timing_end()
    for k in (Q.QLORA_KERNEL_QUANTIZE, Q.QLORA_KERNEL_LORA_GEMM):
        kt[k] = kt2[k]
    elapsed_ms = dp.max_over_ranks(start.elapsed_time(end), dev)
    ms_per_step = elapsed_ms / args.steps
    flops_step = fwd_bwd_flops(M, N, K, r)
    value = flops_step * world / (ms_per_step * 1e-3) / 1e12
    t_fwd = statistics.mean(e[0].elapsed_time(e[1]) for e in evs) * 1e-3
    t_bwd = statistics.mean(e[1].elapsed_time(e[2]) for e in evs) * 1e-3

    kernels = kernel_rooflines(kt, M, N, K, r, peaks)
    # the roofline line is the kernel with the largest share of device time
    dominant = max(kernels, key=lambda k: kernels[k]["total_ms"])
    d = kernels[dominant]
    roofline = {"bound": d["bound"], "achieved": d["achieved"], "peak": d["peak"],
                "unit": d["unit"], "frac": d["frac"], "traffic": TRAFFIC.get(dominant),
                "kernel": dominant, "avg_launch_us": d["avg_us"],
                "algorithmic_per_launch": d["algorithmic_per_launch"],
                "peak_kind": d["peak_kind"]}

    # end to end: every step copies its inputs in from pinned host memory and
    # its results out to pinned host memory.  The copies run on their own
    # streams (one per direction), so that the next step's upload and the
    # previous step's download overlap this step's compute; two device slots
    # alternate, each reused only after its step's results have left.
    e2e = None
    if not args.no_e2e:
        in_keys, out_keys = ("W", "A", "B", "X", "dY"), ("Y", "dX", "dA", "dB")
        slots = sets[:2]
        host_in = [{k: getattr(sl, k).cpu().pin_memory() for k in in_keys} for sl in slots]
        host_out = [{k: torch.empty_like(getattr(sl, k), device="cpu").pin_memory()
                     for k in out_keys} for sl in slots]
        h2d = sum(t.numel() * t.element_size() for t in host_in[0].values())
        d2h = sum(t.numel() * t.element_size() for t in host_out[0].values())
        compute = torch.cuda.current_stream()
        up, down = torch.cuda.Stream(), torch.cuda.Stream()

        def e2e_steps(n):
            up.wait_stream(compute)
            done_compute, done_down = [], []
            for i in range(n):
                j = i % 2
                sl = slots[j]
                with torch.cuda.stream(up):
                    if i >= 2:  # the slot's previous step has computed and downloaded
                        up.wait_event(done_compute[i - 2])
                        up.wait_event(done_down[i - 2])
                    for k, t in host_in[j].items():
                        getattr(sl, k).copy_(t, non_blocking=True)
                    uploaded = torch.cuda.Event()
                    uploaded.record(up)
                compute.wait_event(uploaded)
                run_step(sl, shape, Q, world=world)
                ev = torch.cuda.Event()
                ev.record(compute)
                done_compute.append(ev)
                with torch.cuda.stream(down):
                    down.wait_event(ev)
                    for k, t in host_out[j].items():
                        t.copy_(getattr(sl, k), non_blocking=True)
                    ev2 = torch.cuda.Event()
                    ev2.record(down)
                    done_down.append(ev2)
            compute.wait_stream(up)
            compute.wait_stream(down)

        e2e_steps(args.warmup)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(compute)
        e2e_steps(args.steps)
        e1.record(compute)
        torch.cuda.synchronize()
        e2e_ms = dp.max_over_ranks(e0.elapsed_time(e1), dev) / args.steps
        e2e = {"value": round(flops_step * world / (e2e_ms * 1e-3) / 1e12, 3), "unit": UNIT,
               "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h,
               "path": "pinned host -> device copies (upload stream), qlora_quantize + "
                       "qlora_linear_fwd + qlora_linear_bwd through the C ABI, device -> pinned "
                       "host copies (download stream); two device slots, so that copies of "
                       "neighbouring steps overlap the compute"}

    decode = None
    if rank == 0 and world == 1 and not args.no_decode:
        decode = time_decode(Q, WL, dev, peaks)
    merge = None
    if rank == 0 and world == 1 and not args.no_decode:
        merge = time_merge(Q, sets, shape, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_oracle_sample(shape, CPU_TOKENS, WL)

    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    wb = nf4_bytes(N, K)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,.) tensors of the workload's shapes)",
        "config": workload_config(world),
        "launch": "one CUDA graph of the timed steps" if use_graph else "eager",
        "nf4_weight_gbs": round(2 * wb / (t_fwd + t_bwd) / 1e9, 1),
        "fwd_ms": round(t_fwd * 1e3, 4), "bwd_ms": round(t_bwd * 1e3, 4),
        "fwd_tflops": round(fwd_flops(M, N, K, r) / t_fwd / 1e12, 2),
        "bwd_tflops": round((fwd_bwd_flops(M, N, K, r) - fwd_flops(M, N, K, r)) / t_bwd / 1e12, 2),
        "frac_of_bf16_peak": round(value / world / peaks["bf16_sustained"], 4),
        "roofline": roofline, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches, "clocks": clk.summary(), "decode": decode, "merge": merge,
        "peaks": peaks,
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------- other workloads -------

CONFIGS = {  # --workload name: (workload, linear indices, tokens, input sets, description)
    "single_256": ("single_256", [0], 16, 3,
                   "single linear 256x256 fp32 W, r=8 alpha=16, 16 tokens"),
    "mlp_8192": ("mlp_11008", [0, 1], 8192, 2,
                 "7B MLP gate/up 4096->11008 and down 11008->4096, r=64 alpha=16, 8192 tokens"),
    "stack_7b_layer": ("stack_7b", list(range(7)), 2048, 2,
                       "one layer of the 7B stack (q,k,v,o 4096^2, gate/up 11008x4096, down "
                       "4096x11008), r=16 alpha=32, 2048 tokens; the stack is 32 such layers"),
    "stack_65b_layer": ("stack_65b", list(range(7)), 2048, 2,
                        "one layer of the 65B-shaped stack (8192^2 x4, 22016x8192 x2, "
                        "8192x22016), r=64 alpha=16, 2048 tokens; the stack is 80 such layers"),
}


def run_config(args):
    """One step over the linears of a workload: quantise all, forward in
    order, backward in reverse order (layer-by-layer chaining)."""
    from bit_nf4_quantized_17_b200 import dp
    from bit_nf4_quantized_17_b200 import qlora as Q
    from bit_nf4_quantized_17_b200 import workloads as WL

    name, idx, M, n_sets, desc = CONFIGS[args.workload]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = measured_peaks()
    shapes = [WL.WORKLOADS[name].linears[j] for j in idx]
    sets = [[InputSet(sh, M, WL.stack_seed(0, j) + 1000 * i, 0, dev, Q, WL, dp)
             for sh, j in zip(shapes, idx)] for i in range(n_sets)]
    flops = sum(fwd_bwd_flops(M, sh.d_out, sh.d_in, sh.r) for sh in shapes)
    fused_f = sum(fwd_flops(M, sh.d_out, sh.d_in, sh.r) for sh in shapes)
    fused_b = sum(2 * M * sh.d_out * sh.d_in + 2 * M * sh.d_in * sh.r for sh in shapes)

    def step(group):
        for s, sh in zip(group, shapes):
            Q.qlora_quantize(s.W, out=s.q, workspace=s.qws, check=False)
        for s, sh in zip(group, shapes):
            Q.qlora_linear_fwd(s.q, s.A, s.B, sh.alpha, s.X, Y=s.Y, U_save=s.U, workspace=s.fws)
        for s, sh in reversed(list(zip(group, shapes))):
            Q.qlora_linear_bwd(s.q, s.A, s.B, sh.alpha, s.X, s.U, s.dY, dX=s.dX, dA=s.dA,
                               dB=s.dB, workspace=s.bws)

    for i in range(args.warmup):
        step(sets[i % n_sets])
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clk:
        torch.cuda.synchronize()
        Q.qlora_timing_begin((Q.QLORA_KERNEL_FUSED_FWD, Q.QLORA_KERNEL_FUSED_DGRAD),
                             max_launches=4 * len(shapes) * args.steps)
        start.record()
        for i in range(args.steps):
            step(sets[i % n_sets])
        end.record()
        torch.cuda.synchronize()
        kt = Q.qlora_timing_end()
    ms = start.elapsed_time(end) / args.steps
    value = flops / (ms * 1e-3) / 1e12
    t_f = kt[Q.QLORA_KERNEL_FUSED_FWD][0] / args.steps * 1e-3
    t_b = kt[Q.QLORA_KERNEL_FUSED_DGRAD][0] / args.steps * 1e-3
    nf4 = sum(nf4_bytes(sh.d_out, sh.d_in) for sh in shapes)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,.) tensors of the workload's shapes)",
        "config": {"workload": f"{args.workload}: {desc}; step = quantise + fwd + bwd of "
                               "every linear", "global_batch": M,
                   "l2": f"{n_sets} rotating input sets"},
        "frac_of_bf16_peak": round(value / peaks["bf16_sustained"], 4),
        "fused_fwd_tflops": round(fused_f / t_f / 1e12, 2) if t_f > 0 else None,
        "fused_dgrad_tflops": round(fused_b / t_b / 1e12, 2) if t_b > 0 else None,
        "fused_share": round((t_f + t_b) / (ms * 1e-3), 4),
        "nf4_weight_gbs": round(2 * nf4 / (ms * 1e-3) / 1e9, 1),
        "clocks": clk.summary(), "peaks": peaks,
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------ reference arm ----

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    from threadpoolctl import threadpool_info

    import oracle
    from bit_nf4_quantized_17_b200 import workloads as WL

    shape = WL.WORKLOADS[WORKLOAD].linears[0]
    ms = CPU_TOKENS
    inp = WL.linear_inputs(shape, ms, 0)
    W = inp["W"].float().numpy()
    f = lambda t: t.float().numpy()
    A, B, X, dY = f(inp["A"]), f(inp["B"]), f(inp["X"]), f(inp["dY"])

    def step():
        qt = oracle.quantize(W, 64, 256)
        w_hat = oracle.dequantize(qt).reshape(W.shape)
        oracle.linear_fwd(w_hat, A, B, shape.alpha, X)
        oracle.linear_bwd(w_hat, A, B, shape.alpha, X, dY)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    t = (time.perf_counter() - t0) / args.steps
    flops = fwd_bwd_flops(ms, shape.d_out, shape.d_in, shape.r)
    value = flops / t / 1e12
    cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    sample = (f"oracle quantise of the full 4096x4096 W + fwd/bwd on {ms} of the {TOKENS} "
              f"tokens per step; FLOPs of those tokens / time")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,.) tensors of the workload's shapes)",
        "config": workload_config(world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="launch the timed steps one call at a time instead of one CUDA graph")
    ap.add_argument("--workload", default=WORKLOAD, choices=[WORKLOAD] + sorted(CONFIGS),
                    help="another workload of the problem (one GPU, our arm only)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.workload != WORKLOAD:
        run_config(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
