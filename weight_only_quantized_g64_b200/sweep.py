"""Per-shape timing of the quantized products, and one-call runs for profilers.

    python -m weight_only_quantized_g64_b200.sweep --shapes 2048x2048,3x2048x2048 --Ms 1,16
    python -m weight_only_quantized_g64_b200.sweep --shapes 4096x16384 --Ms 1 --once

A shape is `NxK` (one projection, rq_gemv_wq for M <= 32, rq_gemm_wq above)
or `3xNxK` (three projections of one x, rq_rkv_fused).  Each timed shape
cycles through enough weight copies that one pass reads more than the L2
(about 400 MB), captures the calls in a CUDA graph and times graph replays
with CUDA events; it prints one JSON line per (shape, M, PDL setting).
`--once` makes one call per shape and M with a single weight copy, which is
the launch a profiler should capture.
"""
from __future__ import annotations

import argparse
import json

import torch

from . import build as rq_build
from . import rq, synth


def parse_shape(sh: str):
    parts = [int(t) for t in sh.split("x")]
    if len(parts) not in (2, 3) or (len(parts) == 3 and parts[0] != 3):
        raise ValueError(f"shape {sh!r}: expected NxK or 3xNxK")
    return (3 if len(parts) == 3 else 1), parts[-2], parts[-1]


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--shapes", default="2048x2048,3x2048x2048,8192x2048,2048x8192")
    ap.add_argument("--Ms", default="1,16,32")
    ap.add_argument("--bits", type=int, default=4, choices=(4, 8))
    ap.add_argument("--total-mb", type=int, default=400)
    ap.add_argument("--iters", type=int, default=200)
    ap.add_argument("--pdl", default="1", help="comma list of 0/1")
    ap.add_argument("--once", action="store_true")
    ap.add_argument("--decode-kernel", default="auto", choices=sorted(rq.DECODE_KERNELS),
                    help="kernel of the decode products (M <= 32)")
    ap.add_argument("--product", default="auto", choices=("auto", "gemm"),
                    help="gemm: time rq_gemm_wq at every M (single projections only)")
    a = ap.parse_args(argv)
    rq_build.build()
    rq.lib()
    rq.set_decode_kernel(a.decode_kernel)
    for sh in a.shapes.split(","):
        nmat, N, K = parse_shape(sh)
        per = synth.algorithmic_weight_bytes(N, K, a.bits) * nmat
        copies = 1 if a.once else max(2, int(a.total_mb * 1e6 // per) + 1)
        ws = []
        for c in range(copies + (2 if nmat == 3 and copies == 1 else 0)):
            W = synth.weights(N, K, seed=synth.seed_for(9, c), device="cuda")
            ws.append(rq.quantize_g64(W, a.bits))
            del W
        nw = len(ws)
        for M in [int(t) for t in a.Ms.split(",")]:
            x = synth.activations(M, K, seed=synth.seed_for(9, 0, 1), device="cuda")
            ys = [torch.empty((M, N), dtype=torch.float32, device="cuda") for _ in range(3)]

            if nmat == 3:
                kind = "rkv_fused"
            elif M <= rq.MAX_DECODE_M and a.product == "auto":
                kind = "gemv_wq"
            else:
                kind = "gemm_wq"

            def run():
                for i in range(copies):
                    if nmat == 3:
                        j = [(i + t) % nw for t in range(3)]
                        rq.rkv_fused(x, ws[j[0]], ws[j[1]], ws[j[2]], N, a.bits, ys=ys)
                    elif M <= rq.MAX_DECODE_M and a.product == "auto":
                        rq.gemv_wq(x, ws[i][0], ws[i][1], N, a.bits, y=ys[0])
                    else:
                        rq.gemm_wq(x, ws[i][0], ws[i][1], N, a.bits, y=ys[0])

            for pdl in [int(t) for t in a.pdl.split(",")]:
                rq.set_pdl(bool(pdl))
                run()
                torch.cuda.synchronize()
                if a.once:
                    continue
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    run()
                for _ in range(3):
                    g.replay()
                torch.cuda.synchronize()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                reps = max(1, a.iters // copies)
                e0.record()
                for _ in range(reps):
                    g.replay()
                e1.record()
                torch.cuda.synchronize()
                ms = e0.elapsed_time(e1) / (reps * copies)
                print(json.dumps({"shape": sh, "M": M, "bits": a.bits, "pdl": pdl,
                                  "product": kind, "decode_kernel": a.decode_kernel,
                                  "us": ms * 1e3, "GB/s": per / ms / 1e6, "MB": per / 1e6}),
                      flush=True)
                del g
    st = rq.read_device_status()
    if st != 0:
        raise SystemExit(f"device status {rq.STATUS.get(st, st)}")


if __name__ == "__main__":
    main()
