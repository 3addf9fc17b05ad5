"""Benchmark of the NVFP4 FlashAttention forward on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step is one pass of the whole path over one batch of the workload: amax
and NVFP4 quantisation of Q, K and V, then the fused attention forward (one
fp4_attn_fwd call). value = algorithmic FLOPs (4*B*H*N^2*D, halved when causal)
of all ranks / the slowest rank's device time. Under torchrun (N > 1 ranks) the
heads are sharded: the job is N times the workload's (batch, key/value head)
units, each rank owns one workload-sized slab of them (weak scaling), and a step
is fp4_attn_fwd_sharded: the three tensor maxima of the rank's shard, one NCCL
all-reduce (MAX) of those three floats, quantisation with the global maxima and
the fused forward, so codes match a single-GPU run over the whole job.
Inputs are seeded synthetic tensors; the default workload is the video-DiT
latent grid (B1 H24 N32760 D128). e2e: the same metric through the C-ABI call
on host buffers (fp4_attn_fwd_host), one call per step: the step's q, k, v
copied in from pinned host memory, the forward, the output copied back, all in
the timed region. e2e_pipelined: a stream of batches through
fp4_attn_fwd_host_many, copies overlapped with the neighbouring steps' compute.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FP4 attention fwd TFLOPS at 1 B200 and % of dense FP4 tensor peak"
FP4_DATASHEET_TFLOPS = 9000.0  # NVIDIA B200 dense FP4, no sparsity
L2_BYTES = 126 * 1024 * 1024
# DRAM bytes (read + write) of one attention-kernel launch on the full video-DiT
# workload, from the ncu capture of this kernel (dram__bytes_read.sum +
# dram__bytes_write.sum, one pass). They hold only for the kernel source they
# were taken on, identified by its hash; otherwise traffic is reported null.
ATTN_TRAFFIC = {"workload": "video_dit", "bytes": 170.20e6 + 156.22e6,
                # sha256 of attn_fwd.cuh's code (comments and whitespace removed)
                "attn_fwd_code_sha256":
                    "83dc2c541c6eaab115900f668031c738cb213908cd55762f552e0dc57e138321"}


def code_sha256(path: str) -> str:
    """sha256 of a C++ source with its comments and whitespace removed: the
    traffic figure stays valid across comment-only edits, not code edits."""
    import re
    with open(path) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return hashlib.sha256(" ".join(src.split()).encode()).hexdigest()


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="video_dit")
    ap.add_argument("--impl", default="fp4attn", choices=["fp4attn", "reference"])
    ap.add_argument("--variant", default="exp", choices=["exp", "efq", "fp8pv", "smooth", "bwd"],
                    help="P generation: exp-then-quantize (the default path), EFQ-Softmax, "
                         "or exp-then-quantize to FP8 with V in FP8 (PV as an FP8 contraction); "
                         "smooth: the default path with Q and K smoothed; bwd: the FP4 attention "
                         "backward (one GPU; its own metric)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--heads", type=int, default=0,
                    help="override H and Hkv (keeping their ratio) for a smaller profiling case")
    ap.add_argument("--cpu-rows", type=int, default=0,
                    help="query rows in the oracle's timed sample (0: one per head)")
    return ap.parse_args()


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return m, "MEASURED_PEAKS.json"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, \
            "fallback"


class Clocks:
    """nvidia-smi samples (every 200 ms) while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index, self.proc = index, None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if getattr(self, "lines", None) is not None and self.proc is None:
            return
        self.lines = []
        if self.proc:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
            self.proc = None

    def summary(self):
        mhz, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                maxes.append(float(f[2]))
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max(maxes),
                "reasons": sorted(reasons), "samples": len(mhz)}


def flush_l2(buf):
    buf.add_(1)


def oracle_flags(variant: str) -> int:
    import oracle
    return {"exp": 0, "efq": oracle.FLAG_EFQ, "fp8pv": oracle.FLAG_FP8PV,
            "smooth": oracle.FLAG_SMOOTH_K | oracle.FLAG_SMOOTH_Q}[variant]


def cpu_baseline(wl, q, k, v, rows_total: int, variant: str = "exp"):
    """The oracle, as it stands, on a bounded sample: `rows_total` seeded query
    rows spread over the heads (plus the quantisation of K and V it needs)."""
    import numpy as np
    import oracle
    import synth
    oracle.build()
    per_head = max(1, rows_total // (wl.B * wl.H))
    rows = synth.sample_rows(wl, per_head)
    threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    oracle.attn_fwd(q, k, v, causal=wl.causal, rows=rows, threads=threads,
                    flags=oracle_flags(variant))
    dt = time.perf_counter() - t0
    keys = (rows[:, 2] + 1).astype(np.float64) if wl.causal else np.full(len(rows), wl.N, np.float64)
    flops = float((4.0 * wl.D * keys).sum())
    return {"value": flops / dt / 1e12, "unit": "TFLOPS", "cores": threads, "kind": "oracle",
            "sample": f"{len(rows)} seeded query rows ({per_head} per head) of {wl.name}, "
                      f"plus quantising all of K and V; {dt:.1f} s",
            "seconds": dt}


def run_reference(args, wl):
    """The reference arm: the CPU oracle on a bounded sample per step."""
    if args.variant == "bwd":
        raise SystemExit("the reference arm times the forward; bench --variant bwd reports the "
                         "oracle backward as its cpu_baseline")
    import numpy as np
    import synth
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    synth.build()
    q, k, v = synth.workload_inputs(wl)
    rows_total = args.cpu_rows or wl.B * wl.H
    times, res = [], None
    for i in range(args.warmup + args.steps):
        res = cpu_baseline(wl, q, k, v, rows_total, args.variant)
        if i >= args.warmup:
            times.append(res["seconds"])
    flops = res["value"] * res["seconds"] * 1e12
    val = flops / statistics.mean(times) / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOPS",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": statistics.mean(times) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64/f32 (CPU oracle)",
            "data": "synthetic", "config": {**wl.describe(), "sample": res["sample"]},
            "cpu_baseline": {k2: res[k2] for k2 in ("kind", "cores", "sample")} | {"value": val},
            "e2e": {"value": val, "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_bwd(args, wl):
    """The FP4 attention backward on one GPU: fp4_attn_bwd timed with inputs
    resident (lse from fp4_attn_fwd_lse), e2e through host buffers."""
    import numpy as np
    import torch
    import bit_attention_transformers_b200 as fa
    import synth
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--variant bwd runs on one GPU")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    fa.lib()
    synth.build()
    hq, hk, hv = (torch.empty(shape, dtype=torch.bfloat16, pin_memory=True) for shape in
                  ((wl.B, wl.H, wl.N, wl.D), (wl.B, wl.Hkv, wl.N, wl.D), (wl.B, wl.Hkv, wl.N, wl.D)))
    synth.workload_inputs(wl, outs=[t.view(torch.int16).numpy().view(np.uint16) for t in (hq, hk, hv)])
    hdo = torch.empty_like(hq).pin_memory()
    hdo.view(torch.int16).numpy().view(np.uint16)[...] = synth.normal_bf16(
        hq.numel(), seed=wl.seed + 17, stream=5).reshape(hq.shape)
    q, k, v, do = (t.to(dev) for t in (hq, hk, hv, hdo))
    out, lse = fa.fp4_attn_fwd_lse(q, k, v, causal=wl.causal)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        fa.fp4_attn_bwd(q, k, v, out, do, lse, causal=wl.causal, dq=dq, dk=dk, dv=dv)

    def timed(fn, n):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for a, b in evs:
            flush_l2(flush)
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in evs]

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    fa.fp4_status()
    with Clocks(0) as clk:
        ms = timed(step, args.steps)
    fa.fp4_status()
    ms_per_step = sum(ms) / len(ms)
    fwd_flops = wl.flops
    value = 2.5 * fwd_flops / (ms_per_step * 1e-3) / 1e12
    # the kernels' own tensor work, 8 contractions of 2 N^2 D per head: the dq
    # kernel's S, dP and its two dQ sums (P (dP - c) K^ and P K^) and the dk/dv
    # kernel's dP, dV, dK in bf16, and its S^T in NVFP4 (4x the bf16 rate, so
    # counted as a quarter of a bf16 contraction against the bf16 peak)
    tensor_flops = 7.25 * fwd_flops / 2
    peaks, src = measured_peaks()
    hlse = torch.empty(lse.shape, dtype=torch.float32, pin_memory=True)
    hlse.copy_(lse)
    hout = torch.empty(out.shape, dtype=torch.bfloat16, pin_memory=True)
    hout.copy_(out)
    hdq, hdk, hdv = (torch.empty(t.shape, dtype=torch.bfloat16, pin_memory=True)
                     for t in (dq, dk, dv))

    def e2e():
        gq, gk, gv, go, gdo, gl = (t.to(dev, non_blocking=True)
                                   for t in (hq, hk, hv, hout, hdo, hlse))
        a, b, c = fa.fp4_attn_bwd(gq, gk, gv, go, gdo, gl, causal=wl.causal)
        hdq.copy_(a, non_blocking=True)
        hdk.copy_(b, non_blocking=True)
        hdv.copy_(c, non_blocking=True)
        stream.synchronize()

    e2e()
    e_ms = timed(e2e, max(1, args.steps // 2))
    e_val = 2.5 * fwd_flops / (sum(e_ms) / len(e_ms) * 1e-3) / 1e12
    line = {
        "metric": "FP4 attention bwd TFLOPS at 1 B200 (2.5 x forward FLOPs)", "value": value,
        "unit": "TFLOPS", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4 scores, bf16 gradient contractions",
        "data": "synthetic",
        "config": {**wl.describe(), "pass": "backward (fp4_attn_bwd)", "parallelism": "1 GPU",
                   "l2": "L2 flushed (252 MB write) before every timed step"},
        "roofline": {"bound": "tensor", "achieved": tensor_flops / (ms_per_step * 1e-3) / 1e12,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": tensor_flops / (ms_per_step * 1e-3) / 1e12 / peaks["bf16_tflops"],
                     "traffic": None,
                     "peak_source": f"measured dense bf16 ({src}); the whole call, 7 bf16 "
                                    "contractions of 2 N^2 D per head and one NVFP4 one "
                                    "counted as 1/4; fraction of measured"},
        "e2e": {"value": e_val, "unit": "TFLOPS",
                "h2d_bytes_per_step": (hq.numel() + hk.numel() + hv.numel() + hout.numel()
                                       + hdo.numel()) * 2 + hlse.numel() * 4,
                "d2h_bytes_per_step": (hdq.numel() + hdk.numel() + hdv.numel()) * 2},
        # amax, Q and K codes (2), Q scale regrouping, Q^ and K^ decode (2), V^ decode,
        # dO pad/transpose, lse pad, dq kernel, dk/dv kernel
        "gpu_launches": 11 * args.steps,
    }
    c = clk.summary()
    if c:
        line["clocks"] = c
    if not args.no_cpu_baseline:
        import oracle
        oracle.build()
        rows = synth.sample_rows(wl, max(1, (args.cpu_rows or wl.B * wl.H) // (wl.B * wl.H)))
        a = [t.view(torch.int16).numpy().view(np.uint16) for t in (hq, hk, hv, hdo)]
        t0 = time.perf_counter()
        oracle.attn_bwd(*a, wl.causal, q_rows=rows, kv_rows=np.zeros((0, 3), np.int64))
        dt = time.perf_counter() - t0
        keys = (rows[:, 2] + 1).astype(np.float64) if wl.causal else np.full(len(rows), wl.N, np.float64)
        line["cpu_baseline"] = {"value": 2.5 * float((4.0 * wl.D * keys).sum()) / dt / 1e12,
                                "unit": "TFLOPS", "cores": os.cpu_count() or 1, "kind": "oracle",
                                "sample": f"dq of {len(rows)} seeded query rows of {wl.name} "
                                          f"(plus decoding K, V for them); {dt:.1f} s"}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    import synth
    wl = synth.WORKLOADS[args.workload]
    if args.heads:
        import dataclasses
        g = wl.H // wl.Hkv
        wl = dataclasses.replace(wl, H=args.heads, Hkv=max(1, args.heads // g))
    if args.impl == "reference":
        run_reference(args, wl)
        return
    if args.variant == "bwd":
        run_bwd(args, wl)
        return

    import numpy as np
    import torch
    import torch.distributed as dist
    import bit_attention_transformers_b200 as fa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    fa.lib()

    synth.build()
    shape_q = (wl.B, wl.H, wl.N, wl.D)
    shape_kv = (wl.B, wl.Hkv, wl.N, wl.D)
    hq = torch.empty(shape_q, dtype=torch.bfloat16, pin_memory=True)
    hk = torch.empty(shape_kv, dtype=torch.bfloat16, pin_memory=True)
    hv = torch.empty(shape_kv, dtype=torch.bfloat16, pin_memory=True)
    # rank r holds units r*B*Hkv .. (r+1)*B*Hkv - 1 of the job: its own heads, its own data
    synth.workload_inputs(wl, seed=wl.seed + 7919 * rank,
                          outs=[t.view(torch.int16).numpy().view(np.uint16) for t in (hq, hk, hv)])
    q, k, v = hq.to(dev), hk.to(dev), hv.to(dev)
    out = torch.empty_like(q)
    qf, kf, vf, outf = (t.view(-1, wl.N, wl.D) for t in (q, k, v, out))
    efq, fp8pv = args.variant == "efq", args.variant == "fp8pv"
    smooth = (fa.FP4_SMOOTH_K | fa.FP4_SMOOTH_Q) if args.variant == "smooth" else 0
    ws = fa.workspace(wl.B, wl.H, wl.Hkv, wl.N, wl.D, dev, fp8pv, smooth)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    flops = wl.flops

    def step():
        if world > 1:
            fa.fp4_attn_fwd_sharded(qf, kf, vf, causal=wl.causal, out=outf, efq=efq,
                                    fp8pv=fp8pv, smooth=smooth)
        else:
            fa.fp4_attn_fwd(q, k, v, causal=wl.causal, out=out, ws=ws, efq=efq, fp8pv=fp8pv,
                            smooth=smooth)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def timed(fn, n):
        """Device time (ms) of each of n calls of fn, L2 flushed before each."""
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for s, e in evs:
            flush_l2(flush)
            s.record(stream)
            fn()
            e.record(stream)
        torch.cuda.synchronize()
        return [s.elapsed_time(e) for s, e in evs]

    for _ in range(args.warmup):
        step()
    fa.fp4_status()
    barrier()
    # clocks sampled from the timed steps through the kernel-only and the
    # end-to-end timing below (10 steps alone last ~0.1 s, under one sample)
    clk = Clocks(local).__enter__()
    import atexit
    atexit.register(clk.__exit__, None, None, None)  # the sampler ends even if the run fails
    step_ms = timed(step, args.steps)
    barrier()
    fa.fp4_status()
    total_ms = sum(step_ms)
    if world > 1:
        t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    ms_per_step = total_ms / args.steps
    value = world * flops / (ms_per_step * 1e-3) / 1e12

    # the fused attention kernel alone (same inputs, already quantised)
    vq = fa.fp4_quantize_fp8(v) if fp8pv else fa.fp4_quantize(v, fa.FP4_BLOCK_ALONG_N_T)
    if smooth:
        kmean = fa.fp4_channel_mean(k, fa.fp4_amax(k))
        qmean = fa.fp4_channel_mean(q, fa.fp4_amax(q))
        kq = fa.fp4_quantize_smoothed(k, kmean, fa.fp4_amax_smoothed(k, kmean))
        qq = fa.fp4_quantize_smoothed(q, qmean, fa.fp4_amax_smoothed(q, qmean))
        bias = fa.fp4_score_bias(qmean, k, kmean, wl.H, qq.amax, kq.amax)
    else:
        qq = fa.fp4_quantize(q, fa.FP4_BLOCK_ALONG_D)
        kq = fa.fp4_quantize(k, fa.FP4_BLOCK_ALONG_D)

    def kernel():
        if smooth:
            fa.fp4_attn_fwd_quantized_bias(qq, kq, vq, bias, wl.B, wl.H, wl.Hkv, causal=wl.causal,
                                           out=out)
        else:
            fa.fp4_attn_fwd_quantized(qq, kq, vq, wl.B, wl.H, wl.Hkv, causal=wl.causal, out=out,
                                      efq=efq, fp8pv=fp8pv)

    for _ in range(args.warmup):
        kernel()
    k_ms = statistics.mean(timed(kernel, args.steps))
    fa.fp4_status()

    # end to end: pinned host inputs -> device -> fp4_attn_fwd -> host output
    hout = torch.empty(shape_q, dtype=torch.bfloat16, pin_memory=True)

    def e2e():
        if world > 1:
            for d, h in ((q, hq), (k, hk), (v, hv)):
                d.copy_(h, non_blocking=True)
            fa.fp4_attn_fwd_sharded(qf, kf, vf, causal=wl.causal, out=outf, efq=efq,
                                    fp8pv=fp8pv, smooth=smooth)
            hout.copy_(out, non_blocking=True)
            stream.synchronize()
        else:
            fa.fp4_attn_fwd_host(hq, hk, hv, causal=wl.causal, out=hout, device=dev, efq=efq,
                                 fp8pv=fp8pv, smooth=smooth)

    houts = [hout, torch.empty(shape_q, dtype=torch.bfloat16, pin_memory=True)]
    n_e2e = max(2, args.steps)
    e_pipe = None
    if world > 1:
        for _ in range(max(1, args.warmup // 2)):
            e2e()
        barrier()
        e_ms = timed(e2e, max(1, args.steps // 2))
        barrier()
    else:
        # one C-ABI call per step (copies in, forward, copy out), L2 flushed between
        for _ in range(2):
            e2e()
        e_ms = timed(e2e, n_e2e)
        # a stream of batches through the public host API: each step copies its
        # inputs in and its output out, overlapped with the neighbouring steps'
        # compute
        batches = [(hq, hk, hv)] * n_e2e
        fa.fp4_attn_fwd_host_many(batches[:2], houts, causal=wl.causal, device=dev, efq=efq,
                                  fp8pv=fp8pv, smooth=smooth)
        _, total = fa.fp4_attn_fwd_host_many(batches, [houts[i % 2] for i in range(n_e2e)],
                                             causal=wl.causal, device=dev, efq=efq,
                                             fp8pv=fp8pv, smooth=smooth, return_ms=True)
        e_pipe = flops / (total / n_e2e * 1e-3) / 1e12
    e_total = sum(e_ms)
    if world > 1:
        t = torch.tensor([e_total], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e_total = float(t.item())
    e2e_value = world * flops / (e_total / len(e_ms) * 1e-3) / 1e12
    clk.__exit__(None, None, None)
    fa.fp4_status()

    peaks, src = measured_peaks()
    # dense FP4 = 4x dense bf16 (nominal 9 vs 2.25 PF); with FP8 P and V half the
    # flops (PV) run at FP8's 2x: the time-weighted peak is 1 / (0.5/4 + 0.5/2) = 8/3 x
    peak_ratio = 8.0 / 3.0 if fp8pv else 4.0
    fp4_peak = peak_ratio * peaks["bf16_tflops"]
    achieved = flops / (k_ms * 1e-3) / 1e12
    traffic = None
    kernel_src = os.path.join(ROOT, "bit_attention_transformers_b200", "csrc", "attn_fwd.cuh")
    if (wl.name == ATTN_TRAFFIC["workload"] and not args.heads and args.variant == "exp" and
            code_sha256(kernel_src) == ATTN_TRAFFIC["attn_fwd_code_sha256"]):
        traffic = ATTN_TRAFFIC["bytes"]
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (P and V: e4m3)" if fp8pv else "nvfp4",
        "data": "synthetic",
        "config": {**wl.describe(),
                   "p_generation": {"exp": "exp-then-quantize", "efq": "EFQ-Softmax",
                                    "fp8pv": "exp-then-quantize to FP8 E4M3, V in FP8 E4M3",
                                    "smooth": "exp-then-quantize, Q and K smoothed"}[
                                        args.variant],
                   "parallelism": (f"heads sharded over {world} ranks ({world} x B*Hkv units, "
                                   "one all-reduce MAX of 3 floats per step)") if world > 1
                   else "1 GPU",
                   "l2": "inputs larger than L2 (bf16 Q/K/V of "
                         f"{(hq.numel() + 2 * hk.numel()) * 2 / 1e6:.0f} MB); "
                         "L2 also flushed (252 MB write) before every timed step"},
        "pct_of_fp4_peak": {"value": 100.0 * value / world / FP4_DATASHEET_TFLOPS,
                            "peak_tflops": FP4_DATASHEET_TFLOPS,
                            "peak": "9 PFLOP/s dense FP4, NVIDIA B200 datasheet"},
        "attn_kernel_ms": k_ms,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": fp4_peak,
                     "unit": "TFLOP/s", "frac": achieved / fp4_peak, "traffic": traffic,
                     "peak_source": f"{peak_ratio:.3g} x measured dense bf16 "
                                    f"({peaks['bf16_tflops']} TFLOP/s, "
                                    f"{src}); fraction of measured"},
        "e2e": {"value": e2e_value, "unit": "TFLOPS",
                "h2d_bytes_per_step": (hq.numel() + hk.numel() + hv.numel()) * 2,
                "d2h_bytes_per_step": hout.numel() * 2,
                "how": ("fp4_attn_fwd_host (C ABI): one host-to-host call per step"
                        if world == 1 and not (efq or fp8pv or smooth) else
                        "host copies on the compute stream, then the device entry, one step "
                        "at a time")},
        # per step: amax (1, or 3 when sharded), 3 quantisations, the fused forward;
        # smoothing adds per smoothed tensor the sums, the means and the smoothed
        # maximum, plus Q's score correction
        "gpu_launches": ((7 if world > 1 else 5) + (7 if smooth else 0)) * args.steps,
    }
    if e_pipe is not None:
        line["e2e_pipelined"] = {"value": e_pipe, "unit": "TFLOPS",
                                 "how": "fp4_attn_fwd_host_many: a stream of batches, step i+1's "
                                        "copies in and step i-1's copy out overlapped with step "
                                        "i's compute"}
    c = clk.summary()
    if c:
        line["clocks"] = c
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = {k2: v2 for k2, v2 in
                                cpu_baseline(wl, hq.view(torch.int16).numpy().view(np.uint16),
                                             hk.view(torch.int16).numpy().view(np.uint16),
                                             hv.view(torch.int16).numpy().view(np.uint16),
                                             args.cpu_rows or wl.B * wl.H,
                                             args.variant).items()
                                if k2 != "seconds"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
