#!/usr/bin/env python3
"""Benchmark: decode weight GB/s (and prefill TFLOP/s) of group-64 quantized
RWKV-7 projections on B200, through librq's C ABI.

Default workload: the 13.3B-shaped int4 g64 decode stack -- 61 RWKV-7 layers
of width D = 4096, each with fused R/K/V (3 x 4096^2), O 4096^2, channel-mix
key 4096->16384 and value 16384->4096 -- at every batch M in {1, 2, 4, 8, 16,
32}.  One step = one decode pass through the 61-layer projection stack at each
M (6 x 61 x 4 kernel launches), replayed from CUDA graphs.  The weights
(6.52 GB of codes and scales per pass) are far larger than L2, so every step
streams them from HBM.  `--workload 2` / `3` run the 1.5B-shaped int4 and the
2.9B-shaped int8 stacks instead.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
  python bench.py --case gemv|rkv|gemm|quantize|quantize_ex2 --shape NxK --M m [--bits b]

`--case` runs one product (or quantizer) call per repeat on a single weight
copy with nothing timed: the launch a profiler captures (`ncu -k ... -s 1`
skips the first, warm-up call).

Prints one JSON line (rank 0).  With N > 1 (torchrun) every rank decodes its
own batch through its own copy of the stack (independent replicas, no
collective on the data path: weak scaling); value = bytes all ranks streamed
/ the slowest rank's time.
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from weight_only_quantized_g64_b200 import build as rq_build  # noqa: E402
from weight_only_quantized_g64_b200 import rq, synth  # noqa: E402

METRIC = "decode w4g64 GEMV weight GB/s (% of B200 HBM peak); prefill TFLOP/s; 1 GPU"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

# DRAM traffic of the decode kernels: dram__bytes_read.sum +
# dram__bytes_write.sum of a one-launch ncu capture of the row-block kernel on
# 16384 x 4096 int4 at M = 1, divided by that launch's algorithmic bytes
# (codes + scales).  Traffic grows in proportion to the weights a launch
# streams, so the bench reports this ratio times its average algorithmic bytes
# per launch.  It is valid only for the kernel code it was taken on: when the
# code's hash (comments and whitespace ignored) differs, the bench reports
# traffic as null until a new capture is taken.
DECODE_SOURCES = ("rq_api.cu", "rq_gemv.cu", "rq_gemv_ck.cu", "rq_gemv_unit.cuh", "rq_ptx.cuh",
                  "rq_internal.h", "rq_gemv_rb.cuh", "rq_gemv_rb.cu", "rq_gemv_rb_g64_4.cu",
                  "rq_gemv_rb_g64_8.cu", "rq_tcs.cu")
KERNEL_NAMES = {"rowtile": "gemv_wq_kernel (row tiles)", "cluster": "gemv_ck_kernel (cluster split-K)",
                "rowblock": "gemv_rb_kernel (row blocks)", "tensor": "tcs_kernel (tcgen05, K split over a cluster)"}
DECODE_TRAFFIC = {"code_sha256_16": "9bba2ce732bb77a5", "dram_per_algorithmic_byte": 35697920 / 35651584}


def decode_code_hash():
    import hashlib
    import re
    h = hashlib.sha256()
    for f in DECODE_SOURCES:
        with open(os.path.join(ROOT, "weight_only_quantized_g64_b200", "csrc", f)) as fh:
            text = fh.read()
        text = re.sub(r"//[^\n]*", "", text)
        h.update("".join(text.split()).encode())
    return h.hexdigest()[:16]


def decode_traffic(algorithmic_bytes_per_launch):
    if decode_code_hash() != DECODE_TRAFFIC["code_sha256_16"]:
        return None
    return DECODE_TRAFFIC["dram_per_algorithmic_byte"] * algorithmic_bytes_per_launch


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(
            d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


# ------------------------------------------------------------ distributed --

def dist_setup(n_gpus):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v, world):
    """The largest of every rank's v (device times are taken as the max over
    ranks); the reduction runs where the process group's backend does."""
    if world == 1:
        return v
    dev = "cpu" if torch.distributed.get_backend() == "gloo" else "cuda"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_gbs(world, bytes_per_rank_step, steps, max_ms):
    """Whole-job weight GB/s: the bytes every rank streamed over the slowest
    rank's time (each rank runs its own copy of the stack: weak scaling)."""
    return world * bytes_per_rank_step * steps / (max_ms / 1e3) / 1e9


# ---------------------------------------------------------------- clocks --

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"rq_clocks_bench_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [t.strip() for t in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        busy = [s for s, p in zip(sm, power) if p > 200] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# ------------------------------------------------------------ the stack --

def flush_l2(buf):
    buf.add_(1)   # write a buffer larger than L2


class DecodeStack:
    """Quantized projection weights of every layer of a workload."""

    def __init__(self, wl, rank):
        self.wl = wl
        self.layers = []
        D = wl.projs[0].N
        self.D = D
        for layer in range(wl.layers):
            q = {}
            for pi, pj in enumerate(wl.projs):
                W = synth.weights(pj.N, pj.K, seed=synth.seed_for(wl.index, layer, pi) + 7919 * rank,
                                  device="cuda")
                q[pj.name] = (rq.quantize_g64(W, wl.bits), pj)
                del W
            self.layers.append(q)
        torch.cuda.synchronize()
        self.bytes_per_pass = wl.layers * sum(
            synth.algorithmic_weight_bytes(p.N, p.K, wl.bits) for p in wl.projs)
        self.launches_per_pass = wl.layers * 4

    def kernels(self):
        """{decode kernel: [launch names]} that one pass at each M runs on."""
        wl, out = self.wl, {}
        shapes = [("rkv", wl.projs[0], 3), ("o", wl.projs[3], 1), ("key", wl.projs[4], 1),
                  ("value", wl.projs[5], 1)]
        for M in wl.Ms:
            for name, p, nmat in shapes:
                k = rq.decode_kernel_for(M, p.K, p.N, wl.bits, nmat)
                out.setdefault(k, []).append(f"{name}@M{M}")
        return out

    def buffers(self, M):
        wl = self.wl
        D = self.D
        F = wl.projs[4].N
        xs = {"xD": synth.activations(M, D, seed=100 + M, device="cuda",
                                      massive_channel=wl.massive_channel),
              "xF": synth.activations(M, F, seed=200 + M, device="cuda",
                                      massive_channel=wl.massive_channel)}
        ys = {n: torch.empty((M, p.N), dtype=torch.float32, device="cuda") for n, p in
              ((p.name, p) for p in wl.projs)}
        return xs, ys

    def run_pass(self, xs, ys):
        bits = self.wl.bits
        D = self.D
        for q in self.layers:
            (wr, _), (wk, _), (wv, _) = q["r"], q["k"], q["v"]
            rq.rkv_fused(xs["xD"], wr, wk, wv, D, bits, ys=(ys["r"], ys["k"], ys["v"]))
            (wo, po) = q["o"]
            rq.gemv_wq(xs["xD"], wo[0], wo[1], po.N, bits, y=ys["o"])
            (wkey, pkey) = q["ffn_key"]
            rq.gemv_wq(xs["xD"], wkey[0], wkey[1], pkey.N, bits, y=ys["ffn_key"])
            (wval, pval) = q["ffn_value"]
            rq.gemv_wq(xs["xF"], wval[0], wval[1], pval.N, bits, y=ys["ffn_value"])


def capture(fn):
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()           # warm (sets kernel attributes outside capture)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


# ---------------------------------------------------------- CPU baseline --

def oracle_threads(rows):
    """OpenMP threads the oracle runs with: one per host core, but no more than
    the rows it parallelises over (set before the oracle library loads)."""
    threads = max(1, min(os.cpu_count() or 1, rows))
    os.environ["OMP_NUM_THREADS"] = str(threads)
    return threads


def cpu_oracle_rate(wl, budget_s=12.0, layer_rows=None):
    """The oracle, as it stands, on a bounded sample of the decode workload:
    `layer_rows` rows (default: one per host core, at least 16) of every
    projection of layer 0 at every M, repeated until `budget_s` of wall time;
    returns (weight GB/s, threads used, sample)."""
    if layer_rows is None:
        layer_rows = max(16, os.cpu_count() or 1)
    cores = oracle_threads(layer_rows)
    import oracle
    oracle.build()
    jobs = []
    for pi, pj in enumerate(wl.projs):
        W = synth.weights(layer_rows, pj.K, seed=synth.seed_for(wl.index, 0, pi))
        c, s, _ = oracle.quantize_g64(W.numpy(), wl.bits)
        for M in wl.Ms:
            x = synth.activations(M, pj.K, seed=M, massive_channel=wl.massive_channel).numpy()
            jobs.append((x, c, s, synth.algorithmic_weight_bytes(layer_rows, pj.K, wl.bits)))
    done_bytes, t0, reps = 0, time.perf_counter(), 0
    while True:
        for x, c, s, b in jobs:
            oracle.matmul(x, c, s, wl.bits, with_bound=False)
            done_bytes += b
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    sample = (f"oracle fp64 products of {layer_rows} rows of each of the {len(wl.projs)} "
              f"projections of one layer at M in {list(wl.Ms)}, {reps} repetitions "
              f"({dt:.1f} s)")
    return done_bytes / dt / 1e9, cores, sample


def reference_arm(args, wl, rank, world):
    """`--impl reference`: the oracle timed on the host cores, rank 0 only."""
    if rank != 0:
        return
    rows = max(4, os.cpu_count() or 1)   # the oracle parallelises over rows
    cores = oracle_threads(rows)
    import oracle
    oracle.build()
    jobs = []
    for pi, pj in enumerate(wl.projs):
        W = synth.weights(rows, pj.K, seed=synth.seed_for(wl.index, 0, pi))
        c, s, _ = oracle.quantize_g64(W.numpy(), wl.bits)
        for M in wl.Ms:
            x = synth.activations(M, pj.K, seed=M, massive_channel=wl.massive_channel).numpy()
            jobs.append((x, c, s, synth.algorithmic_weight_bytes(rows, pj.K, wl.bits)))
    step_bytes = sum(j[3] for j in jobs)

    def step():
        for x, c, s, _ in jobs:
            oracle.matmul(x, c, s, wl.bits, with_bound=False)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = step_bytes * args.steps / dt / 1e9
    sample = (f"each step: oracle fp64 products of {rows} rows of each projection of one "
              f"layer at M in {list(wl.Ms)}")
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": wl.name, "bits": wl.bits, "M": list(wl.Ms)},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------ prefill, quantizer --

def bench_prefill(hbm_peak, tf_peak, reps=50):
    wl = synth.WORKLOADS[4]
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")  # 256 MB
    weights = []
    for pi, pj in enumerate(wl.projs):
        W = synth.weights(pj.N, pj.K, seed=synth.seed_for(4, 0, pi), device="cuda")
        weights.append((rq.quantize_g64(W, 4), pj))
        del W
    per_layer = {"d_x_d": 4, "ffn_key": 1, "ffn_value": 1}
    out = {}
    s = torch.cuda.current_stream()
    for M in wl.Ms:
        tot_flops, tot_ms = 0.0, 0.0
        shapes = {}
        for (cw, pj) in weights:
            x = synth.activations(M, pj.K, seed=M, device="cuda")
            y = torch.empty((M, pj.N), dtype=torch.float32, device="cuda")
            rq.gemm_wq(x, cw[0], cw[1], pj.N, 4, y=y)   # warm
            times = []
            for _ in range(reps):
                flush_l2(flush)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(s)
                rq.gemm_wq(x, cw[0], cw[1], pj.N, 4, y=y)
                e1.record(s)
                e1.synchronize()
                times.append(e0.elapsed_time(e1))
            ms = statistics.median(times)
            fl = 2.0 * M * pj.N * pj.K
            shapes[pj.name] = {"ms": ms, "tflops": fl / ms / 1e9}
            tot_flops += fl * per_layer[pj.name]
            tot_ms += ms * per_layer[pj.name]
        tf = tot_flops / tot_ms / 1e9
        out[str(M)] = {"tflops_layer": tf, "frac": tf / tf_peak, "shapes": shapes}
    return out


def bench_quantizer(hbm_peak, reps=50):
    N, K = 16384, 4096
    W = synth.weights(N, K, seed=5, device="cuda")
    codes, scales = rq.empty_weights(N, K, 4)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    rq.quantize_g64(W, 4, codes=codes, scales=scales)
    s = torch.cuda.current_stream()
    times = []
    for _ in range(reps):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        rq.quantize_g64(W, 4, codes=codes, scales=scales)
        e1.record(s)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    byts = N * K * 4 + synth.algorithmic_weight_bytes(N, K, 4)
    # the E[x^2]-weighted scale search on the same shape, 7 candidates
    # (offline work; also reads E[x^2] and writes the choices)
    e2 = torch.rand(K, generator=torch.Generator(device="cuda").manual_seed(6), device="cuda") * 4.0
    factors = torch.tensor([1.0, 0.95, 0.9, 0.85, 0.8, 0.75, 0.7], device="cuda")
    rq.quantize_g64_ex2(W, e2, 4, factors, codes=codes, scales=scales)
    t2 = []
    for _ in range(max(5, reps // 5)):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        rq.quantize_g64_ex2(W, e2, 4, factors, codes=codes, scales=scales)
        e1.record(s)
        e1.synchronize()
        t2.append(e0.elapsed_time(e1))
    ms2 = statistics.median(t2)
    return {"shape": [N, K], "bits": 4, "ms": ms, "gbs": byts / ms / 1e6,
            "frac": byts / ms / 1e6 / hbm_peak,
            "e2_search": {"candidates": 7, "ms": ms2, "gbs": byts / ms2 / 1e6,
                          "frac": byts / ms2 / 1e6 / hbm_peak}}


def bench_gptq(reps=3):
    """GPTQ on one 4096 x 4096 projection (int4 g64) with 512 synthetic
    calibration tokens: device time of each step (hessian, factor, column
    loop), median of `reps` runs.  Offline work: reported, not a headline."""
    N = K = 4096
    T = 512
    g = torch.Generator(device="cuda")
    g.manual_seed(17)
    X = torch.randn((T, K), generator=g, device="cuda").to(torch.float16)
    W0 = synth.weights(N, K, seed=18, device="cuda")
    s = torch.cuda.current_stream()
    out = {"hessian": [], "factor": [], "loop": []}
    for _ in range(reps):
        W = W0.clone()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        ev[0].record(s)
        H = rq.gptq_hessian(X)
        ev[1].record(s)
        U, dead = rq.gptq_factor(H)
        ev[2].record(s)
        rq.gptq_g64(W, 4, U, dead)
        ev[3].record(s)
        ev[3].synchronize()
        for i, k in enumerate(("hessian", "factor", "loop")):
            out[k].append(ev[i].elapsed_time(ev[i + 1]))
        del H, U, dead, W
    res = {k: statistics.median(v) for k, v in out.items()}
    res.update({"shape": [N, K], "tokens": T, "bits": 4, "unit": "ms",
                "loop_tflops": N * K * K / (res["loop"] / 1e3) / 1e12})
    return res


# ------------------------------------------------------- profiling case --

def run_case(args):
    """One call per repeat of a single product or quantizer on one weight
    copy, synchronised after each call; nothing is timed or printed but a
    status line.  The launch a profiler captures."""
    rq_build.build()
    torch.cuda.set_device(0)
    rq.lib()
    N, K = (int(t) for t in args.shape.split("x"))
    W = synth.weights(N, K, seed=5, device="cuda")
    if args.case == "quantize":
        for _ in range(args.repeat):
            rq.quantize_g64(W, args.bits)
            torch.cuda.synchronize()
    elif args.case == "gptq":
        X = synth.activations(512, K, seed=8, device="cuda")
        for _ in range(args.repeat):
            U, dead = rq.gptq_factor(rq.gptq_hessian(X))
            rq.gptq_g64(W.clone(), args.bits, U, dead)
            torch.cuda.synchronize()
    elif args.case == "quantize_ex2":
        e2 = synth.activations(64, K, seed=6, device="cuda").float().pow(2).mean(0)
        factors = torch.tensor([1.0, 0.95, 0.9, 0.85, 0.8, 0.75, 0.7], device="cuda")
        for _ in range(args.repeat):
            rq.quantize_g64_ex2(W, e2, args.bits, factors)
            torch.cuda.synchronize()
    else:
        w = rq.quantize_g64(W, args.bits)
        del W
        x = synth.activations(args.M, K, seed=7, device="cuda")
        rq.set_decode_kernel(args.decode_kernel)
        for _ in range(args.repeat):
            if args.case == "gemv":
                rq.gemv_wq(x, w[0], w[1], N, args.bits)
            elif args.case == "rkv":
                rq.rkv_fused(x, w, w, w, N, args.bits)
            else:
                rq.gemm_wq(x, w[0], w[1], N, args.bits)
            torch.cuda.synchronize()
    print(f"case {args.case} {args.shape} M={args.M} bits={args.bits} x{args.repeat}: ok "
          f"(device status {rq.read_device_status(reset=True)})", flush=True)


# ------------------------------------------------------------------ main --

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", type=int, default=5, choices=[2, 3, 5])
    ap.add_argument("--case", default=None,
                    choices=["gemv", "rkv", "gemm", "quantize", "quantize_ex2", "gptq"],
                    help="one call per repeat of a single product or quantizer (profiling target)")
    ap.add_argument("--shape", default="4096x4096", help="NxK of --case")
    ap.add_argument("--M", type=int, default=1, help="batch of --case")
    ap.add_argument("--bits", type=int, default=4, choices=[4, 8], help="bits of --case")
    ap.add_argument("--repeat", type=int, default=2, help="calls of --case")
    ap.add_argument("--decode-kernel", default="auto", choices=sorted(rq.DECODE_KERNELS),
                    help="decode kernel of --case gemv/rkv")
    ap.add_argument("--no-pdl", action="store_true")
    ap.add_argument("--skip-extras", action="store_true",
                    help="decode only (no prefill/quantizer/cpu baseline/e2e)")
    args = ap.parse_args()
    if args.case is not None:
        run_case(args)
        return
    wl = synth.WORKLOADS[args.workload]

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        reference_arm(args, wl, rank, world)
        return

    assert args.warmup >= 3, "at least 3 warm-up steps"
    rq_build.build()
    rank, world, local = dist_setup(args.gpus)
    rq.lib()
    rq.set_pdl(not args.no_pdl)
    hbm_peak, tf_peak, tf_sust, peak_kind = peaks()

    stack = DecodeStack(wl, rank)
    graphs, bufs = {}, {}
    for M in wl.Ms:
        xs, ys = stack.buffers(M)
        bufs[M] = (xs, ys)
        graphs[M] = capture(lambda xs=xs, ys=ys: stack.run_pass(xs, ys))

    s = torch.cuda.current_stream()
    for _ in range(args.warmup):
        for M in wl.Ms:
            graphs[M].replay()
    torch.cuda.synchronize()

    # ---- timed region: K steps, each = one pass per M -----------------
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(s)
    for _ in range(args.steps):
        for M in wl.Ms:
            graphs[M].replay()
    t_end.record(s)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), world)

    # per-M split of the same passes (events between replays, no host sync)
    n_split = max(20, args.steps // 10)
    marks = [[torch.cuda.Event(enable_timing=True) for _ in range(len(wl.Ms) + 1)]
             for _ in range(n_split)]
    for st in range(n_split):
        marks[st][0].record(s)
        for i, M in enumerate(wl.Ms):
            graphs[M].replay()
            marks[st][i + 1].record(s)
    torch.cuda.synchronize()
    per_m_ms = {M: sum(marks[st][i].elapsed_time(marks[st][i + 1]) for st in range(n_split))
                for i, M in enumerate(wl.Ms)}

    bytes_per_step = stack.bytes_per_pass * len(wl.Ms)
    launches_per_step = stack.launches_per_pass * len(wl.Ms)
    ms_per_step = elapsed_ms / args.steps
    value = job_gbs(world, bytes_per_step, args.steps, elapsed_ms)
    per_rank_gbs = bytes_per_step / (ms_per_step / 1e3) / 1e9
    per_m = {str(M): {"us_per_pass": per_m_ms[M] / n_split * 1e3,
                      "gbs": stack.bytes_per_pass / (per_m_ms[M] / n_split / 1e3) / 1e9,
                      "frac": stack.bytes_per_pass / (per_m_ms[M] / n_split / 1e3) / 1e9 / hbm_peak}
             for M in wl.Ms}

    # ---- e2e: host inputs in, host results out, through the same calls --
    e2e = None
    if not args.skip_extras:
        host_x = {M: {k: v.cpu().pin_memory() for k, v in bufs[M][0].items()} for M in wl.Ms}
        host_y = {M: {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
                      for k, v in bufs[M][1].items()} for M in wl.Ms}
        h2d = sum(t.numel() * t.element_size() for M in wl.Ms for t in host_x[M].values())
        d2h = sum(t.numel() * t.element_size() for M in wl.Ms for t in host_y[M].values())
        e2e_steps = max(10, args.steps // 10)
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(e2e_steps):
            for M in wl.Ms:
                xs, ys = bufs[M]
                for k in xs:
                    xs[k].copy_(host_x[M][k], non_blocking=True)
                graphs[M].replay()
                for k in ys:
                    host_y[M][k].copy_(ys[k], non_blocking=True)
        e1.record(s)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
        e2e = {"value": job_gbs(world, bytes_per_step, e2e_steps, e2e_ms), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_ms / e2e_steps,
               "how": "pinned host x -> device, replay of the captured rq_* calls, "
                      "every output -> pinned host, per step"}

    prefill = quant = cpu = gptq = None
    if not args.skip_extras:
        prefill = bench_prefill(hbm_peak, tf_peak)
        quant = bench_quantizer(hbm_peak)
        gptq = bench_gptq()
        if rank == 0 and world == 1:
            g, cores, sample = cpu_oracle_rate(wl)
            cpu = {"value": g, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample}

    if rank == 0:
        achieved = per_rank_gbs
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16xint4->f32" if wl.bits == 4 else "f16xint8->f32",
            "data": "synthetic (seeded N(0,0.02^2) weights quantized on device, N(0,1) fp16 x)",
            "config": {"workload": wl.name, "bits": wl.bits, "layers": wl.layers,
                       "M": list(wl.Ms), "bytes_per_pass": stack.bytes_per_pass,
                       "l2": "weights (%.0f MB per pass) larger than L2; no flush needed"
                             % (stack.bytes_per_pass / 1e6),
                       "pdl": not args.no_pdl, "graphs": True, "parallelism": f"replicas{world}"},
            "hbm_frac": value / world / hbm_peak,
            "per_M": per_m,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved / hbm_peak,
                         "traffic": decode_traffic(bytes_per_step / launches_per_step),
                         "kernel": "decode products (fused RKV + O + key + value, all M): " +
                                   ", ".join(f"{KERNEL_NAMES[k]} x{len(v)}" for k, v in
                                             sorted(stack.kernels().items())),
                         "bytes_per_launch": bytes_per_step / launches_per_step,
                         "us_per_launch": ms_per_step * 1e3 / launches_per_step,
                         "peak_kind": peak_kind + " copy bandwidth"},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
            "prefill": prefill,
            "prefill_peak": {"tflops": tf_peak, "kind": peak_kind + " bf16 (fp16 same nominal rate)"},
            "quantizer": quant,
            "gptq": gptq,
        }
        print(json.dumps(line), flush=True)

    for g in graphs.values():
        del g
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
