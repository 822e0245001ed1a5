"""Where the tensor-core expert GEMMs wait (the routed call of a prefill layer).

    python -m bit_expert_ffn_fp32_b200.build --trace
    python -m bit_expert_ffn_fp32_b200.trace_prefill [WORKLOAD] [--calls N]

Loads libmoe_trace.so (built with -DMOE_TC_TRACE), runs the routed expert call
of the layer N times on fresh tokens with the L2 evicted before each call, and
prints for each kernel and role (producer warp 0, epilogue warp 8, the MMA
thread) the median over CTAs and calls of the cycles spent in each wait, as a
share of that role's run time.
"""
from __future__ import annotations

import argparse
import ctypes as C
import os

import numpy as np
import torch

from . import configs, native, synth
from .layer import MoEStack, x_tensor

ROLES = ("producer", "epilogue", "mma", "tma")
SLOTS = {  # role -> slot -> meaning
    "producer": {1: "packed codes landed", 2: "A slot free (MMA done)", 4: "dequantise + TMEM store + arrive",
                 3: "of which tcgen05.st issue", 5: "of which tcgen05.wait::st"},
    "epilogue": {1: "accumulator full (tfull)", 2: "TMEM loads (gate/up)"},
    "mma": {1: "A stage full", 2: "B stage full", 3: "accumulator free (tempty)"},
    "tma": {1: "code slot free (producers done)", 3: "issuing code loads"},
}


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("workload", nargs="?", default="prefill_T8192_d2048_E512_k10_f768_q2")
    ap.add_argument("--calls", type=int, default=5)
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
    tl.moe_tc_trace_read.restype = C.c_int
    tl.moe_tc_trace_read.argtypes = [C.c_void_p]
    wl = configs.WORKLOADS[args.workload]
    stack = MoEStack(wl)
    T, k, E, d, f = wl.T, wl.k, wl.E, wl.d, wl.f
    b = stack.buffers(T)
    flush = torch.empty(512 << 18, dtype=torch.float32, device="cuda")
    buf = np.zeros(2 * 256 * 4 * 8, np.uint64)
    per = {(kk, r): [] for kk in range(2) for r in range(4)}
    for it in range(args.calls + 1):
        x = x_tensor(synth.gen_x(wl.seed, 0, T, d, stream=it))
        native.route(x, stack.Wr[0], stack.bias[0], T, d, E, k, b.logits, b.idx, b.w, b.status)
        native.permute(b.idx, T, k, E, b.counts, b.offsets, b.sorted_tok, b.sorted_j, b.inv, b.active, b.perm_ws,
                       0 if b.perm_ws is None else b.perm_ws.numel(), b.status)
        flush.fill_(1.0)
        torch.cuda.synchronize()
        tl.moe_tc_trace_read(buf.ctypes.data)          # clear
        native.expert_ffn(stack.qpool, stack.slot_of[0], x, T, d, f, E, k, b.offsets, b.sorted_tok, b.sorted_j,
                          b.active, None, b.y_perm, b.h_ws, b.h_ws.numel(), b.status)
        torch.cuda.synchronize()
        if tl.moe_tc_trace_read(buf.ctypes.data) != 0:
            raise SystemExit("trace read failed")
        if it == 0:
            continue
        tr = buf.reshape(2, 256, 4, 8).astype(np.int64)
        for kk in range(2):
            for r in range(4):
                rows = tr[kk, :, r, :]
                rows = rows[rows[:, 0] > 0]
                per[(kk, r)].append(rows)
    print(f"{wl.name}: routed expert call, L2 evicted before each call, status {int(b.status.item())}")
    for kk, kname in enumerate(("gate/up", "down")):
        for r, role in enumerate(ROLES):
            rows = np.concatenate(per[(kk, r)])
            tot = np.median(rows[:, 0])
            cnt = np.median(rows[:, 6])
            parts = ", ".join(f"{nm} {100 * np.median(rows[:, s] / rows[:, 0]):.1f}%"
                              for s, nm in SLOTS[role].items())
            unit = {"epilogue": "tiles", "tma": "loads"}.get(role, "stages")
            print(f"  {kname:8s} {role:9s} {tot / 1e3:9.1f} kcycles, {cnt:6.0f} {unit}: {parts}")


if __name__ == "__main__":
    main()
