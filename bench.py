#!/usr/bin/env python
"""Benchmark of the mixed-bitwidth Q-GEMM on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline (one JSON line on rank 0): packed-weight GB/s of the decode call
(M = 1) on the 70B MLP up_proj shape K = 8192, N = 28672 at 2.55 bits per
weight, widths {2,3,4,5,6,8} per 32-row block, random act-order perm, fp16
activations.  One step = one qgemm call.  Steps rotate over enough distinct
weight copies (> 3x the 126 MB L2) that every step streams its weights from
HBM; steps are captured in CUDA graphs and timed with CUDA events on the
launching stream.

Extra objects on the same line:
  roofline      the GEMV kernel against measured HBM bandwidth;
  cpu_baseline  the CPU oracle timed on the host cores (rank 0, N = 1);
  e2e           the same metric through the public call with host buffers
                (x copied in from pinned memory, y copied back, every step);
  prefill       TFLOP/s of the M = 2048 prefill GEMM (K = 8192, N = 28672,
                4.0 bpw, bf16 activations) against the dense tensor peak;
  decode_m_gbs, crossover_sweep, stack (with --full): other M of the headline
                shape, the 8192 x 8192 M sweep that locates the GEMV/GEMM
                crossover, and the 80-layer Llama-3-70B linear stack as tokens/s;
  clocks        SM clocks and throttle reasons sampled during the timed region.

--impl reference times the CPU oracle (the only reference implementation this
method has here) on the same workload, each step a bounded column sample.
Multi-GPU (--gpus N under torchrun): independent replicas, one per GPU, no
collective on the data path (weak scaling); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

HEADLINE = "decode_8192x28672_2p55"
PREFILL = "prefill_2048x8192x28672_4p0"
PREFILL_M = 2048
SWEEP = "sweep_8192x8192_3p75"
SWEEP_MS = (1, 2, 4, 8, 16, 32, 64, 128, 256, 512)
STACK = "llama70b_stack_2p5"
METRIC = "Q-GEMM weight GB/s at M=1 (% of HBM) and TFLOP/s at M=2048 (% of peak)"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ------------------------------------------------------------------ helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sust=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    src="of measured")
    return dict(hbm=FALLBACK_HBM_GBS, bf16=FALLBACK_BF16_TFLOPS, bf16_sust=1400.0, src="of fallback")


def call_bytes(K, N, M, rows, x_bytes=2):
    """Algorithmic bytes of one call: packed words, scales, x, y, perm, schedule."""
    G = (K + 127) // 128
    return 4 * N * rows + 2 * G * N + x_bytes * M * K + 2 * M * N + 4 * K + (K // 32) * 5 + 4


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled in the background."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.samples = []
        self.proc = None
        self.marks = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def mark(self, name):
        self.marks.append((name, time.time()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for ts, line in self.samples:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            rows.append((ts, parts))
        window = [r for r in rows if t0 - 0.05 <= r[0] <= t1 + 0.05]
        where = "timed region"
        if not window:
            window, where = rows, "whole run (timed region shorter than the sampling period)"
        if not window:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(p[1]) for _, p in window if p[1].replace(".", "").isdigit()]
        smax = [float(p[2]) for _, p in window if p[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, p in window for i in range(4)
                          if p[5 + i].lower().startswith("active")})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(window), "window": where}


def dist_setup(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, ws):
    """The largest v over all ranks (device time of the slowest replica)."""
    if ws == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------ GPU problems

class Layer:
    """Device-resident inputs of one Q-GEMM call (weights, scales, schedule)."""

    def __init__(self, w, M, layer=0, matrix=0, device="cuda", x=True):
        import mixed_bitwidth_weight_b200 as q
        if w.matrices:
            _, K, N = w.matrices[matrix]
        else:
            K, N = w.K, w.N
        self.K, self.N, self.M = K, N, M
        bits = W.schedule_for(w, K, layer, matrix)
        offs = W.offsets(bits)
        self.rows = int(offs[-1])
        self.bits = torch.as_tensor(bits, device=device)
        self.offs = torch.as_tensor(offs, device=device)
        self.perm = torch.as_tensor(W.permutation(K, 0, layer, matrix, identity=w.identity_perm),
                                    device=device)
        self.qw = W.words(self.rows, N, 0, layer, matrix, device=device)
        self.scales = W.scales(bits, N, 0, layer, matrix, device=device)
        self.x = W.activations(M, K, 0, layer, matrix, dtype=w.x_dtype, device=device) if x else None
        self.y = torch.empty(M, N, dtype=torch.float16, device=device)
        self.ws = q.workspace(M, K, N, device=device)

    def call(self, q, x=None, y=None):
        q.qgemm(self.x if x is None else x, self.perm, self.qw, self.scales, self.bits, self.offs,
                self.y if y is None else y, self.ws)


def graph_of(fn, n):
    """CUDA graph with n calls of fn(i)."""
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn(0)                                     # untimed warm call outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        for i in range(n):
            fn(i)
    return g


def run_steps(fn, steps, chunk):
    """Replay graphs so that exactly `steps` calls of fn run."""
    graphs = {}

    def get(n):
        if n not in graphs:
            graphs[n] = graph_of(fn, n)
        return graphs[n]

    full, rem = divmod(steps, chunk)
    plan = [chunk] * full + ([rem] if rem else [])
    for n in set(plan):
        get(n)
    return [get(n) for n in plan]


def time_graphs(graphs, ws):
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    e0.record(st)
    for g in graphs:
        g.replay()
    e1.record(st)
    torch.cuda.synchronize()
    t1 = time.time()
    barrier(ws)
    return e0.elapsed_time(e1) / 1e3, t0, t1


def decode_copies(w, M, target_bytes):
    one = call_bytes(w.K, w.N, M, W.target_word_rows(w.K // 32, w.target_bpw) if w.target_bpw
                     else (w.K // 32) * w.uniform_bits)
    return max(1, math.ceil(target_bytes / one))


def bench_decode(q, w, M, steps, warmup, ws, chunk=192):
    """GB/s of one workload at M rows, rotating over copies > 3x L2."""
    R = decode_copies(w, M, 3 * L2_BYTES + 1)
    base = Layer(w, M)
    layers = [base]
    for r in range(1, R):                    # distinct copies of the weights (same values)
        L = Layer.__new__(Layer)
        L.__dict__.update(base.__dict__)
        L.qw = base.qw.clone()
        L.scales = base.scales.clone()
        L.ws = q.workspace(M, base.K, base.N)
        layers.append(L)
    fn = lambda i: layers[i % R].call(q)  # noqa: E731
    wg = run_steps(fn, warmup, chunk)
    tg = run_steps(fn, steps, chunk)
    for g in wg:
        g.replay()
    secs, t0, t1 = time_graphs(tg, ws)
    secs = max_over_ranks(secs, ws)
    nbytes = call_bytes(base.K, base.N, M, base.rows)
    return dict(secs=secs, t0=t0, t1=t1, bytes=nbytes, rows=base.rows, copies=R,
                gbs=nbytes * steps / secs / 1e9, us=secs / steps * 1e6, layer=base)


def bench_prefill(q, w, M, steps, warmup, ws):
    """TFLOP/s of the prefill GEMM, rotating over weight copies > 3x L2."""
    base = Layer(w, M)
    one = 4 * base.N * base.rows + 2 * ((base.K + 127) // 128) * base.N
    R = max(1, math.ceil((3 * L2_BYTES + 1) / one))
    layers = [base]
    for r in range(1, R):
        L = Layer.__new__(Layer)
        L.__dict__.update(base.__dict__)
        L.qw = base.qw.clone()
        L.scales = base.scales.clone()
        layers.append(L)
    fn = lambda i: layers[i % R].call(q)  # noqa: E731
    wg = run_steps(fn, warmup, 16)
    tg = run_steps(fn, steps, 16)
    for g in wg:
        g.replay()
    secs, t0, t1 = time_graphs(tg, ws)
    secs = max_over_ranks(secs, ws)
    flops = 2.0 * M * base.K * base.N
    return dict(secs=secs, t0=t0, t1=t1, flops=flops, rows=base.rows, copies=R,
                tflops=flops * steps / secs / 1e12, ms=secs / steps * 1e3, layer=base)


def bench_sweep(q, w, Ms, ws):
    """Crossover sweep: one shape, several M; GB/s and TFLOP/s per M and the path used."""
    out = {}
    for M in Ms:
        base = Layer(w, M)
        one = call_bytes(base.K, base.N, M, base.rows)
        R = max(1, math.ceil((3 * L2_BYTES + 1) / (4 * base.N * base.rows)))
        layers = [base]
        for r in range(1, R):
            L = Layer.__new__(Layer)
            L.__dict__.update(base.__dict__)
            L.qw = base.qw.clone()
            L.scales = base.scales.clone()
            L.ws = q.workspace(M, base.K, base.N)
            layers.append(L)
        fn = lambda i: layers[i % R].call(q)  # noqa: E731
        n = 400 if M <= 64 else 100
        for g in run_steps(fn, 10, 10):
            g.replay()
        secs, _, _ = time_graphs(run_steps(fn, n, 50), ws)
        secs = max_over_ranks(secs, ws)
        us = secs / n * 1e6
        out[str(M)] = {"path": q.qgemm_path_for(M, base.K, base.N), "us": round(us, 2),
                       "gbs": round(one / us / 1e3, 1),
                       "tflops": round(2.0 * M * base.K * base.N / us / 1e6, 2)}
        del layers, base
        torch.cuda.empty_cache()
    return out


def bench_stack(q, w, steps, ws):
    """The 80-layer linear stack at M = 1: tokens/s = 1 / (time of all calls)."""
    calls = []
    for layer in range(w.layers):
        for mi in range(len(w.matrices)):
            calls.append(Layer(w, 1, layer=layer, matrix=mi))
    total_bytes = sum(call_bytes(c.K, c.N, 1, c.rows) for c in calls)
    fn = lambda i: calls[i % len(calls)].call(q)  # noqa: E731
    n = len(calls) * steps
    for g in run_steps(fn, len(calls), len(calls)):
        g.replay()
    secs, _, _ = time_graphs(run_steps(fn, n, len(calls)), ws)
    secs = max_over_ranks(secs, ws)
    tok_s = steps / secs
    out = {"tokens_per_s": round(tok_s, 2), "calls_per_token": len(calls),
           "bytes_per_token": total_bytes, "gbs": round(total_bytes * tok_s / 1e9, 1)}
    del calls
    torch.cuda.empty_cache()
    return out


def bench_e2e(q, L, steps, warmup, ws):
    """Public call with host buffers: x in from pinned memory, y back, every step."""
    xh = L.x.cpu().pin_memory()
    yh = torch.empty(L.y.shape, dtype=L.y.dtype).pin_memory()
    xd = torch.empty_like(L.x)

    def step():
        xd.copy_(xh, non_blocking=True)
        L.call(q, x=xd)
        yh.copy_(L.y, non_blocking=True)

    for _ in range(max(3, min(warmup, 50))):
        step()
    n = max(1, min(steps, 2000))
    torch.cuda.synchronize()
    barrier(ws)
    t0 = time.perf_counter()
    for _ in range(n):
        step()
    torch.cuda.synchronize()
    secs = max_over_ranks(time.perf_counter() - t0, ws)
    return dict(gbs=L_bytes(L) * n / secs / 1e9, steps=n, h2d=xh.numel() * xh.element_size(),
                d2h=yh.numel() * yh.element_size())


def L_bytes(L):
    return call_bytes(L.K, L.N, L.M, L.rows)


def cpu_baseline(w, M):
    """The oracle as it stands, on the host cores: one full decode call, 3 runs."""
    import oracle
    pr = W.make_problem(w, M)
    qw = pr["words"].numpy().view(np.uint32)
    x = pr["x"].to(torch.float64).numpy()
    times, used = [], 0
    for _ in range(3):
        t = time.perf_counter()
        _, used = oracle.qgemm_f64(x, pr["perm"].numpy(), qw, pr["scales"].numpy(), pr["bits"])
        times.append(time.perf_counter() - t)
    secs = float(np.median(times))
    nbytes = call_bytes(pr["K"], pr["N"], M, int(pr["offs"][-1]))
    return {"value": round(nbytes / secs / 1e9, 4), "unit": "GB/s", "cores": used, "kind": "oracle",
            "sample": f"one full {w.name} call at M={M} (all {pr['N']} columns), median of 3 runs, "
                      f"{secs:.3f} s each"}


def traffic_from_profiles(kernel_tag):
    """dram bytes per launch from a committed ncu summary, if its source digest
    still matches the library sources (else null)."""
    import glob
    try:
        from mixed_bitwidth_weight_b200 import _build
        digest = _build._digest()
    except Exception:  # noqa: BLE001
        return None
    for f in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        txt = open(f).read()
        if f"kernel_tag: {kernel_tag}" not in txt:
            continue
        vals = dict(l.split(":", 1) for l in txt.splitlines() if l.startswith(("traffic_bytes_per_launch:", "source_digest:")))
        if vals.get("source_digest", "").strip() == digest:
            try:
                return float(vals["traffic_bytes_per_launch"])
            except (KeyError, ValueError):
                return None
    return None


# ----------------------------------------------------------------- arms

def run_ours(args):
    ws, rank, local = dist_setup(args)
    import mixed_bitwidth_weight_b200 as q
    w = W.WORKLOADS[HEADLINE]
    M = 1
    pk = peaks()
    sampler = ClockSampler(local)
    if rank == 0 or True:
        sampler.start()
    time.sleep(0.2)
    res = bench_decode(q, w, M, args.steps, args.warmup, ws)
    clocks = sampler.summary(res["t0"], res["t1"])
    wp = W.WORKLOADS[PREFILL]
    pre = bench_prefill(q, wp, PREFILL_M, max(16, min(160, args.steps // 100)), 5, ws)
    pre_clocks = sampler.summary(pre["t0"], pre["t1"])
    extra = {}
    if args.full:
        extra["decode_m_gbs"] = {}
        for m in (2, 4, 8, 16):
            r = bench_decode(q, w, m, min(args.steps, 2000), min(args.warmup, 200), ws)
            extra["decode_m_gbs"][str(m)] = round(r["gbs"], 1)
        extra["crossover_sweep"] = bench_sweep(q, W.WORKLOADS[SWEEP], SWEEP_MS, ws)
        extra["stack"] = bench_stack(q, W.WORKLOADS[STACK], 3, ws)
    e2e = bench_e2e(q, res["layer"], args.steps, args.warmup, ws)
    sampler.stop()
    cpu = cpu_baseline(w, M) if (rank == 0 and ws == 1 and not args.no_cpu) else None
    achieved = res["bytes"] / (res["us"] * 1e-6) / 1e9
    line = {
        "metric": METRIC,
        "value": round(res["gbs"] * ws, 2),
        "unit": "GB/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(res["us"] / 1e3, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16",
        "data": "synthetic (seeded SplitMix64 inputs; random words = uniform codes)",
        "config": {"workload": HEADLINE, "M": M, "K": w.K, "N": w.N,
                   "bpw": round(res["rows"] / (w.K // 32) + 0.125, 4),
                   "weight_copies": res["copies"],
                   "l2": f"inputs larger than L2: {res['copies']} weight copies rotated "
                         f"({res['copies'] * res['bytes'] / 1e6:.0f} MB > 3x 126 MB)",
                   "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm"],
                     "unit": "GB/s", "frac": round(achieved / pk["hbm"], 4),
                     "traffic": traffic_from_profiles("gemv_int_decode_8192x28672_m1"),
                     "kernel": "qg::gemv_int_kernel<1> (+ qg::xprep_int_kernel, overlapped by PDL; "
                               "achieved uses the whole step time)", "peak_source": pk["src"],
                     "bytes_per_launch": res["bytes"]},
        "prefill": {
            "workload": PREFILL, "M": PREFILL_M, "K": wp.K, "N": wp.N,
            "bpw": round(pre["rows"] / (wp.K // 32) + 0.125, 4), "x_dtype": "bf16",
            "mma_dtype": "f16 (x scaled per row by a power of two, exact)",
            "value": round(pre["tflops"] * ws, 2), "unit": "TFLOP/s", "ms_per_call": round(pre["ms"], 4),
            "weight_copies": pre["copies"],
            "roofline": {"bound": "tensor", "achieved": round(pre["tflops"], 1), "peak": pk["bf16"],
                         "unit": "TFLOP/s", "frac": round(pre["tflops"] / pk["bf16"], 4),
                         "peak_sustained": pk["bf16_sust"],
                         "frac_sustained": round(pre["tflops"] / pk["bf16_sust"], 4),
                         "traffic": traffic_from_profiles("gemm_prefill_2048x8192x28672"),
                         "kernel": "qg::gemm_kernel (+ qg::xperm_kernel; achieved uses the whole call)",
                         "peak_source": pk["src"] + " dense bf16 (fp16 runs at the same rate)"},
            "clocks": pre_clocks,
        },
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e["gbs"] * ws, 2), "unit": "GB/s",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "steps": e2e["steps"], "how": "eager qgemm() per step; x H2D from pinned, y D2H to pinned"},
        "gpu_launches": 2 * args.steps,
        "gpu_launches_how": "timed decode region: xprep_int_kernel + gemv_int_kernel per step",
        "clocks": clocks,
    }
    line.update(extra)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_reference(args):
    """The CPU oracle on the headline workload: each step a column sample sized
    so the whole run stays within about a minute."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    w = W.WORKLOADS[HEADLINE]
    M = 1
    pr = W.make_problem(w, M)
    qw = pr["words"].numpy().view(np.uint32)
    x = pr["x"].to(torch.float64).numpy()
    perm, s, bits = pr["perm"].numpy(), pr["scales"].numpy(), pr["bits"]
    N, K, rows = pr["N"], pr["K"], int(pr["offs"][-1])
    t = time.perf_counter()
    oracle.qgemm_f64(x, perm, qw, s, bits, cols=np.arange(256))
    per_col = (time.perf_counter() - t) / 256
    total = args.steps + args.warmup
    ncols = int(max(8, min(N, 60.0 / max(1, total) / per_col)))
    rng = np.random.default_rng(0)
    sample = [np.sort(rng.choice(N, size=ncols, replace=False)) for _ in range(4)]
    used = 0
    for i in range(args.warmup):
        _, used = oracle.qgemm_f64(x, perm, qw, s, bits, cols=sample[i % 4])
    t = time.perf_counter()
    for i in range(args.steps):
        _, used = oracle.qgemm_f64(x, perm, qw, s, bits, cols=sample[i % 4])
    secs = time.perf_counter() - t
    frac = ncols / N
    nbytes = call_bytes(K, N, M, rows) * frac
    val = nbytes * args.steps / secs / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs / max(1, args.steps) * 1e3, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": HEADLINE, "M": M, "K": K, "N": N},
        "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": used, "kind": "oracle",
                         "sample": f"{ncols} of {N} columns per step (bytes scaled by the fraction)"},
        "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_profile_target(args):
    """A few plain calls of one leg, no timing: the command that ncu captures
    (--profile decode | prefill)."""
    import mixed_bitwidth_weight_b200 as q
    torch.cuda.set_device(0)
    if args.profile == "decode":
        L = Layer(W.WORKLOADS[HEADLINE], 1)
    else:
        L = Layer(W.WORKLOADS[PREFILL], PREFILL_M)
    for _ in range(args.profile_calls):
        L.call(q)
    torch.cuda.synchronize()
    err = q.qgemm_device_error(clear=True)
    print(json.dumps({"profile": args.profile, "calls": args.profile_calls, "device_error": err}))
    if err:
        sys.exit(1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=2000)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--full", action="store_true", help="also sweep M and the 80-layer stack")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline")
    ap.add_argument("--profile", choices=["decode", "prefill"], default=None,
                    help="run a few untimed calls of one leg (for ncu) and exit")
    ap.add_argument("--profile-calls", type=int, default=6)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.profile:
        run_profile_target(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
