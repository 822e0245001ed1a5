"""Phase timeline of the one-launch decode layer (moe_layer_decode).

    python -m bit_expert_ffn_fp32_b200.build --trace
    python -m bit_expert_ffn_fp32_b200.trace_decode [WORKLOAD] [--launches N] [--warm]

Loads libmoe_trace.so (the library built with -DMOE_DECODE_TRACE) and runs
the layer (or, for a stacked workload, all layers in one launch, tracing
layer L/2) as the benchmark does: bursts of back-to-back steps on fresh tokens
(resident in HBM), each step after a 512 MiB write and a 256 MiB read of other
buffers (unless --warm), CUDA events around every launch. The trace of the last
launch of each burst is read; the report gives, for each phase boundary, the
median over bursts of the median and the slowest CTA (microseconds since the
first CTA started), the launch time between events and the SM clock the kernel
ran at (cycles over nanoseconds between kernel start and end).
"""
from __future__ import annotations

import argparse
import ctypes as C
import os

import numpy as np
import torch

from . import configs, native, synth
from .layer import MoEStack, x_tensor

POINTS = {12: "x staged", 13: "router rows landed", 1: "logits written", 2: "grid barrier passed",
          14: "top-k: logits loaded", 15: "top-k: threshold rounds", 16: "top-k: candidates gathered",
          17: "top-k: ranked", 3: "top-k + gates", 4: "routing tables", 11: "copies of the first tasks issued",
          **{18 + w: f"task 1 row group landed (warp {w})" for w in range(8)},
          26: "task 1 gate/up computed (warp 0 alone)", 6: "task 1 gate/up computed (all warps)",
          7: "task 1 h exchanged", 27: "task 1 down slice landed (warp 0)",
          28: "task 1 down computed (warp 0 alone)", 8: "task 1 down computed (all warps)",
          9: "task 1 atomics done", 10: "layer end"}


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("workload", nargs="?", default="decode_T1_d2048_E512_k10_f768_q2")
    ap.add_argument("--launches", type=int, default=40)
    ap.add_argument("--warm", action="store_true")
    args = ap.parse_args()
    path = os.path.join(native.PKG, "libmoe_trace.so")
    if not os.path.exists(path):
        raise SystemExit("libmoe_trace.so missing: python -m bit_expert_ffn_fp32_b200.build --trace")
    tl = C.CDLL(path)
    for name, (res, argt) in native.SIGNATURES.items():
        fn = getattr(tl, name)
        fn.restype = res
        fn.argtypes = argt
    native.lib = tl
    wl = configs.WORKLOADS[args.workload]
    stack = MoEStack(wl)
    b = stack.buffers(wl.T)
    wbuf = torch.empty(512 << 18, dtype=torch.float32, device="cuda")
    rbuf = torch.ones(256 << 18, dtype=torch.float32, device="cuda")
    out = torch.empty((), dtype=torch.float32, device="cuda")
    xs = [x_tensor(synth.gen_x(wl.seed, 0, wl.T, wl.d, stream=s), "cuda") for s in range(16)]
    sb = stack.stack_buffers(wl.T) if stack.L > 1 else None
    xst = [torch.stack([x_tensor(synth.gen_x(wl.seed, l, wl.T, wl.d, stream=s), "cuda") for l in range(stack.L)])
           for s in range(4)] if stack.L > 1 else None
    buf = np.zeros(4096 * 32, np.uint64)
    acc = {k: [] for k in POINTS}
    starts, ev, mhz = [], [], []
    burst = 6
    for it in range(args.launches + 3):
        evs = []
        for j in range(burst):
            if not args.warm:
                wbuf.fill_(float(j))
                torch.sum(rbuf, 0, out=out)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            if stack.L > 1:
                stack.forward_stack(xst[0 if args.warm else (it * burst + j) % len(xst)], sb)
            else:
                stack.forward_fused(0, xs[0 if args.warm else (it * burst + j) % len(xs)], b)
            e1.record()
            evs.append((e0, e1))
        torch.cuda.synchronize()
        if it < 3:
            continue
        ev.extend(a.elapsed_time(c) * 1e3 for a, c in evs[1:])
        tl.moe_decode_trace_read(buf.ctypes.data)
        tr = buf.reshape(4096, 32)
        G = int((tr[:, 0] > 0).sum())
        ns = tr[:G, :].astype(np.int64)
        cyc = (ns[:, 31] - ns[:, 30]).astype(np.float64)
        dur = (ns[:, 29] - ns[:, 0]).astype(np.float64)
        mhz.append(float(np.median(cyc / dur * 1e3)))
        ns = ns[:, :29]
        rel = np.where(ns > 0, (ns - ns[:, 0].min()) / 1000.0, np.nan)
        starts.append(float((ns[:, 0].max() - ns[:, 0].min()) / 1000.0))
        for k in POINTS:
            if np.isfinite(rel[:, k]).any():
                acc[k].append((np.nanmedian(rel[:, k]), np.nanmax(rel[:, k])))
    st = int((sb.status if sb is not None else b.status).item())
    print(f"{wl.name}: {G} CTAs, {'warm' if args.warm else 'L2 evicted before each launch'}, status {st}"
          + (f"; layer {stack.L // 2} of {stack.L} traced" if stack.L > 1 else ""))
    print(f"launch time between CUDA events: median {np.median(ev):.2f} us; CTA start spread median "
          f"{np.median(starts):.2f} us; SM clock during the kernel: median {np.median(mhz):.0f} MHz")
    print(f"{'point':34s} {'median CTA':>11s} {'slowest CTA':>12s}  (us since first CTA start)")
    for k, nm in POINTS.items():
        if acc[k]:
            a = np.array(acc[k])
            print(f"{nm:34s} {np.median(a[:, 0]):11.2f} {np.median(a[:, 1]):12.2f}")


if __name__ == "__main__":
    main()
