"""Throughput of one sparse-MoE FFN layer on B200 (C ABI, CUDA kernels).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole layer -- router + top-k, permutation, cache
lookup, routed experts, shared expert, combine -- over one batch of T synthetic
tokens, each step on fresh tokens already resident in HBM. Default workload:
one decode token through a layer of d=2048, 512 experts, top-10 + shared,
f=768, Q2 weights, Zipf-skewed routing, all experts resident.

Timing: CUDA events on the launching stream around every step; a 512 MiB write
between steps evicts the 126 MB L2, so every step reads its weights from HBM.
With N > 1 (torchrun), every rank runs an independent replica on its own
tokens (no collective on the data path); the reported time is the max over
ranks. The expert FFN calls are timed separately for the roofline line.

--impl reference times the CPU oracle (plain C, fp64) on a bounded sample of
the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s (decode T=1/4, 8K prefill); % of HBM / tensor roofline"
FLUSH_BYTES = 512 << 20


def _env_int(name, default):
    v = os.environ.get(name)
    return int(v) if v not in (None, "") else default


# DRAM bytes (read + written) per step of the roofline kernel(s), from one
# ncu capture (dram__bytes_read.sum + dram__bytes_write.sum; see profiles/),
# valid only while the sources it was captured on are unchanged.
PROFILED_TRAFFIC = {
    # fused decode layer kernel, one launch per step
    "decode_T1_d2048_E512_k10_f768_q2": (("decode_layer.cu", "mma_q.cuh", "layout.h", "common.cuh"),
                                         "866ff83c958ad8d0", 20.56e6),
    # expert FFN launches of one step: fp16 gathers, tcgen05 gate/up and down, routed and shared
    "prefill_T8192_d2048_E512_k10_f768_q2": (("ffn_tc05.cu", "tc05.cuh", "layout.h", "common.cuh", "ffn_mma.cu"),
                                             "60d411ce6b0a09e6", 2506e6),
}


def _profiled_traffic(workload: str):
    import hashlib

    entry = PROFILED_TRAFFIC.get(workload)
    if entry is None:
        return None
    files, digest, nbytes = entry
    m = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "bit_expert_ffn_fp32_b200", "csrc", f), "rb") as fh:
            m.update(fh.read())
    return nbytes if m.hexdigest()[:16] == digest else None


def _measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, out_dir: str | None = None):
        """The raw samples go to <out_dir>/clocks_gpu<i>.csv (default: a temporary directory)."""
        import tempfile

        self.gpu = gpu_index
        self.proc = None
        d = out_dir or tempfile.mkdtemp(prefix="moe_clocks_")
        self.path = os.path.join(d, f"clocks_gpu{gpu_index}.csv")

    def start(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "50"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.fh.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as fh:
            for line in fh:
                c = [x.strip() for x in line.split(",")]
                if len(c) < 9:
                    continue
                try:
                    sm.append(float(c[1]))
                    mx = float(c[2])
                except ValueError:
                    continue
                for n, v in zip(names, c[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ reference arm (CPU oracle)
def run_reference(args, wl, rank):
    if rank != 0:
        return 0
    sys.path.insert(0, os.path.join(ROOT, "oracle"))
    import oracle as orc
    from bit_expert_ffn_fp32_b200 import synth
    from bit_expert_ffn_fp32_b200.configs import ZIPF_ALPHA

    Wr = synth.gen_router(wl.seed, 0, wl.E, wl.d)
    rank_p = synth.gen_rank_perm(wl.seed, 0, wl.E)
    bias = synth.zipf_bias(rank_p, ZIPF_ALPHA) if wl.zipf else None
    shared = synth.gen_expert(wl.seed, 0, wl.E, wl.fmt, wl.d, wl.f)
    get = lambda e: synth.gen_expert(wl.seed, 0, e, wl.fmt, wl.d, wl.f)  # noqa: E731
    # Each step is one oracle layer call on a bounded token sample; the run stops
    # after the requested steps or a ~120 s budget, whichever comes first.
    T_s = min(wl.T, 4)
    times = []
    t_start = time.perf_counter()
    for step in range(min(args.warmup, 1) + args.steps):
        x = synth.gen_x(wl.seed, 0, T_s, wl.d, stream=10_000 + step)
        t0 = time.perf_counter()
        orc.layer(x, Wr, bias, get, shared, wl.k, wl.fmt)
        if step >= min(args.warmup, 1):
            times.append(time.perf_counter() - t0)
        if time.perf_counter() - t_start > 120.0 and times:
            break
    tot = sum(times) * wl.layers  # a step of a stacked workload is wl.layers layer calls
    value = T_s * len(times) / tot
    sample = (f"{len(times)} of {args.steps} steps run (120 s budget), {T_s} token(s) of {wl.name} per step, "
              f"oracle layer incl. dequantisation, single thread"
              + (f"; one layer call timed per step, x{wl.layers} for the {wl.layers} layers" if wl.layers > 1 else ""))
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": wl.name, "tokens_per_step": T_s},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline(wl, budget_s=12.0):
    """The oracle as it stands, on a bounded sample of the workload (rank 0, N=1)."""
    sys.path.insert(0, os.path.join(ROOT, "oracle"))
    import oracle as orc
    from bit_expert_ffn_fp32_b200 import synth
    from bit_expert_ffn_fp32_b200.configs import ZIPF_ALPHA

    Wr = synth.gen_router(wl.seed, 0, wl.E, wl.d)
    bias = synth.zipf_bias(synth.gen_rank_perm(wl.seed, 0, wl.E), ZIPF_ALPHA) if wl.zipf else None
    shared = synth.gen_expert(wl.seed, 0, wl.E, wl.fmt, wl.d, wl.f)
    get = lambda e: synth.gen_expert(wl.seed, 0, e, wl.fmt, wl.d, wl.f)  # noqa: E731
    T_s = min(wl.T, 4)
    n_tok, t_tot, it = 0, 0.0, 0
    while t_tot < budget_s and it < 64:
        x = synth.gen_x(wl.seed, 0, T_s, wl.d, stream=20_000 + it)
        t0 = time.perf_counter()
        orc.layer(x, Wr, bias, get, shared, wl.k, wl.fmt)
        t_tot += time.perf_counter() - t0
        n_tok += T_s
        it += 1
    return {"value": n_tok / (t_tot * wl.layers), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{it} oracle layer calls x {T_s} token(s) of {wl.name} ({t_tot:.1f} s, single thread, "
                      f"dequantisation included"
                      + (f"; x{wl.layers} layers per token" if wl.layers > 1 else "") + ")"}


# ------------------------------------------------------------------ host completion of misses
MISS_DTYPE = [("layer", "<i4"), ("expert", "<i4"), ("token", "<i4"), ("j", "<i4"), ("gate", "<f4")]


def _time_host_misses(stack, wl, bufs, x_step):
    """moe_complete_misses_host over one step's miss lists (all layers), the
    missed experts in canonical host storage (generated first, not timed), the
    completion of every layer timed on the host clock with all threads."""
    import time

    from bit_expert_ffn_fp32_b200 import native

    L, T = wl.layers, wl.T
    work, n_rec, n_exp = [], 0, 0
    for l in range(L):
        recs = np.array(stack.misses(bufs[l]), dtype=MISS_DTYPE)
        if len(recs) == 0:
            continue
        y = np.ascontiguousarray(bufs[l].y[:T].cpu().numpy())
        canon = {e: stack.canonical_expert(l, e) for e in sorted(set(recs["expert"].tolist()))}
        work.append((l, recs, y, canon, native.expert_table(wl.E, canon), np.ascontiguousarray(x_step[l])))
        n_rec += len(recs)
        n_exp += len(canon)
    threads = len(os.sched_getaffinity(0))
    t0 = time.perf_counter()
    for l, recs, y, _canon, tab, xl in work:
        native.complete_misses_host(wl.fmt, wl.d, wl.f, tab, wl.E, recs, len(recs), l, xl, T, y, 0)
    dt = time.perf_counter() - t0
    return {"ms_per_step": dt * 1e3, "misses_per_step": n_rec, "distinct_experts_per_step": n_exp,
            "threads": threads, "call": "moe_complete_misses_host (host C++, fp32 lookup-table dot products), "
            "one call per layer", "sample": "the misses of the last end-to-end step"}


# ------------------------------------------------------------------ our arm
def run_ours(args, wl, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from bit_expert_ffn_fp32_b200 import configs, native, replicas, synth
    from bit_expert_ffn_fp32_b200.layer import MoEStack, x_tensor

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    # L > 1 (the stacked-layer workload): a step takes the T tokens through all
    # L layers, each layer with its own seeded input and its own outputs
    L = wl.layers
    stack = MoEStack(wl, device=dev)
    T = wl.T
    bufs = [stack.buffers(T)] + [stack.buffers(T, fresh=True) for _ in range(L - 1)]  # one set per layer
    b = bufs[0]
    stream = torch.cuda.current_stream()
    n_steps = args.warmup + args.steps
    # steps get their own tokens, generated up front and resident in HBM (at most
    # 256 MiB of distinct inputs, cycled; the L2 is evicted between steps anyway)
    n_x = max(1, min(n_steps, (256 << 20) // (L * T * wl.d * 2)))
    xs_host = [np.stack([synth.gen_x(wl.seed, l, T, wl.d, stream=s) for l in range(L)])
               for s in replicas.token_streams(rank, n_x)]
    xs_dev = torch.stack([torch.stack([x_tensor(xl, dev) for xl in x]) for x in xs_host])

    class _Cycle:
        def __getitem__(self, i):
            return xs_dev[i % n_x]

    xs = _Cycle()
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]

    fused = args.path == "fused" or (args.path == "auto" and T <= 8)
    # many tokens: gate-weighted accumulation inside the expert call, no y_perm/combine
    atomic = not fused and args.combine == "atomic"
    if L > 1 and not fused:
        raise SystemExit("a multi-layer workload runs the one-launch decode path (T <= 8)")

    def layer_step(xset, evs=None):
        k, E, d, f = wl.k, wl.E, wl.d, wl.f
        if fused:
            if evs:
                evs[1].record(stream)
            for l in range(L):
                stack.forward_fused(l, xset[l], bufs[l])
            if evs:
                evs[2].record(stream)
            return
        x = xset[0]
        native.route(x, stack.Wr[0], stack.bias[0], T, d, E, k, b.logits, b.idx, b.w, b.status)
        native.permute(b.idx, T, k, E, b.counts, b.offsets, b.sorted_tok, b.sorted_j, b.inv, b.active, b.perm_ws,
                       0 if b.perm_ws is None else b.perm_ws.numel(), b.status)
        native.cache_lookup(stack.slot_of[0], stack.num_slots, 0, b.idx, b.w, b.offsets, b.sorted_tok,
                            b.sorted_j, T, k, E, b.sop, b.miss, b.miss_count, b.idx.numel(), b.status)
        if evs:
            evs[1].record(stream)
        if atomic:  # shared expert writes y, routed experts add gate * y_e into it
            native.expert_ffn(stack.qpool, stack.shared_slot[0], x, T, d, f, 1, 1, b.sh_offsets, b.sh_sorted_tok,
                              b.sh_sorted_j, b.sh_active, None, b.y, b.h_sh, b.h_sh.numel(), b.status)
            native.expert_ffn(stack.qpool, stack.slot_of[0], x, T, d, f, E, k, b.offsets, b.sorted_tok,
                              b.sorted_j, b.active, b.w, b.y, b.h_ws, b.h_ws.numel(), b.status)
            if evs:
                evs[2].record(stream)
            return
        native.expert_ffn(stack.qpool, stack.slot_of[0], x, T, d, f, E, k, b.offsets, b.sorted_tok, b.sorted_j,
                          b.active, None, b.y_perm, b.h_ws, b.h_ws.numel(), b.status)
        native.expert_ffn(stack.qpool, stack.shared_slot[0], x, T, d, f, 1, 1, b.sh_offsets, b.sh_sorted_tok,
                          b.sh_sorted_j, b.sh_active, None, b.y_sh, b.h_sh, b.h_sh.numel(), b.status)
        if evs:
            evs[2].record(stream)
        native.combine(b.y_perm, b.inv, b.w, b.sop, b.y_sh, T, k, d, b.y)

    ffn_launches = 3 if T * wl.k >= 512 and wl.fmt == 2 else 2  # (+ gather on the tensor-core path)
    perm_launches = 1 if native.permute_workspace_bytes(T, wl.k, wl.E) == 0 else 3
    launches_per_step = L if fused else 2 + perm_launches + 1 + 2 * ffn_launches + (0 if atomic else 1)

    # distinct routed experts per step (for the algorithmic bytes), from a warm-up pass
    for s in range(args.warmup):
        flush.fill_(1.0)
        layer_step(xs[s])
    torch.cuda.synchronize()
    for bl in bufs:
        bl.status.zero_()

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank, args.clocks_dir)
    sampler.start()
    time.sleep(0.2)
    for i in range(args.steps):
        flush.fill_(float(i))
        ev[i][0].record(stream)
        layer_step(xs[args.warmup + i])
        ev[i][3].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    step_ms = [ev[i][0].elapsed_time(ev[i][3]) for i in range(args.steps)]
    total_ms = sum(step_ms)
    # The dominant kernel's own time, for the roofline line: the same steps again
    # with events around it (kept out of the timed steps above, whose value they
    # would inflate). With one launch per step it is the step itself.
    if fused:
        ffn_ms = step_ms
    else:
        for i in range(args.steps):
            flush.fill_(float(i))
            layer_step(xs[args.warmup + i], ev[i])
        torch.cuda.synchronize()
        ffn_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(args.steps)]
    status = 0
    for bl in bufs:
        status |= int(bl.status.item())

    # distinct resident experts, resident pairs and misses of each step's routing,
    # summed over the layers (not timed)
    n_act, n_pairs, n_miss = [], [], []
    for i in range(min(args.steps, (256 if T <= 64 else 4) if L == 1 else 8)):
        layer_step(xs[args.warmup + i])
        a_sum = p_sum = m_sum = 0
        for l, bl in enumerate(bufs):
            na = int(bl.active[0].item())
            ids = bl.active[1:1 + na].cpu().numpy()
            a_sum += int((stack.slot_of_host[l][ids] >= 0).sum())
            p_sum += int((bl.sop[: T * wl.k] >= 0).sum().item())
            m_sum += int(bl.miss_count.item())
        n_act.append(a_sum)
        n_pairs.append(p_sum)
        n_miss.append(m_sum)
    mean_act = float(np.mean(n_act))
    res_pairs_mean = float(np.mean(n_pairs))
    hit_rate = res_pairs_mean / (L * T * wl.k)

    total_ms, ffn_total = replicas.max_over_ranks([total_ms, sum(ffn_ms)], device=dev)

    # ---- e2e: pinned host tokens in, layer, result out, every step
    e2e_ms = None
    x_pin = torch.from_numpy(np.stack(xs_host).view(np.int16)).pin_memory()  # [n_x][L][T][d]
    n_y = min(args.steps, max(2, (256 << 20) // (L * T * wl.d * 4)))
    y_pin = torch.empty((n_y, L, T, wl.d), dtype=torch.float32).pin_memory()
    x_dev = torch.empty((L, T, wl.d), dtype=torch.int16, device=dev)
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    for i in range(args.steps):
        flush.fill_(float(i))
        e2e_ev[i][0].record(stream)
        x_dev.copy_(x_pin[i % n_x], non_blocking=True)
        layer_step(x_dev)
        for l in range(L):
            y_pin[i % n_y, l].copy_(bufs[l].y[:T], non_blocking=True)
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = sum(e2e_ev[i][0].elapsed_time(e2e_ev[i][1]) for i in range(args.steps))
    (e2e_ms,) = replicas.max_over_ranks([e2e_ms], device=dev)
    if world > 1:
        dist.barrier()

    if rank != 0:
        return 0
    # stacked layers: the host completion of the last e2e step's misses, on this machine's cores
    host_leg = None
    if L > 1 and not args.no_host_misses:
        host_leg = _time_host_misses(stack, wl, bufs, xs_host[(args.steps - 1) % n_x])
    hbm_peak, tc_peak, peak_kind = _measured_peaks()
    eb = native.expert_bytes(wl.fmt, wl.d, wl.f)
    ffn_bytes = (mean_act + L) * eb                # routed resident experts + the shared experts, read once
    layer_bytes = L * wl.E * wl.d * 4 + ffn_bytes  # + the fp32 router weights (all L layers of a step)
    kern_bytes = layer_bytes if fused else ffn_bytes
    ffn_avg_s = ffn_total / args.steps / 1e3
    achieved = kern_bytes / ffn_avg_s / 1e9
    tensor_bound = not fused and T * wl.k >= 512 and wl.fmt == 2
    ffn_flops = 2.0 * 3 * wl.d * wl.f * (res_pairs_mean + T)   # routed resident pairs + shared, per step
    tokens = world * T * args.steps
    value = replicas.job_throughput(T * args.steps, world, total_ms)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "step_ms_quantiles": {"median": float(np.median(step_ms)), "p90": float(np.percentile(step_ms, 90)),
                              "min": float(np.min(step_ms)), "note": "this rank's per-step CUDA-event times"},
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": ("f16 (dequantised q2) x f16 -> f32" if (not fused and T * wl.k >= 512 and wl.fmt == 2)
                  else "q2xf16->f32" if wl.fmt == 2 else "q3xf16->f32"), "data": "synthetic",
        "config": {"workload": wl.name, "tokens_per_step": T, "l2": "512 MiB write between steps (flushed)",
                   "path": "moe_layer_decode (one launch)" if fused else
                   "step-by-step calls" + (", gate-weighted accumulation in the routed expert call" if atomic else
                                           ", y_perm + moe_combine"),
                   "parallelism": f"replicas x{world}", "layers_per_step": L,
                   "step_algorithmic_bytes": layer_bytes,
                   "step_GBps": layer_bytes / (total_ms / args.steps / 1e3) / 1e9,
                   "mean_distinct_resident_experts": mean_act, "hit_rate": hit_rate,
                   "misses_per_step": float(np.mean(n_miss))},
        "roofline": ({"bound": "tensor",
                      "kernel": "moe_expert_ffn_q2 tcgen05 grouped GEMMs (gate/up + down, routed + shared)",
                      "achieved": ffn_flops / ffn_avg_s / 1e12, "peak": tc_peak, "peak_kind": peak_kind + " bf16 burst",
                      "unit": "TFLOP/s", "frac": ffn_flops / ffn_avg_s / 1e12 / tc_peak,
                      "traffic": _profiled_traffic(wl.name),
                      "flops_per_launch": ffn_flops, "avg_launch_us": ffn_avg_s * 1e6} if tensor_bound else
                     {"bound": "hbm",
                      "kernel": ("decode_layer_kernel (moe_layer_decode: whole layer, one launch per layer)" if fused else
                                 "moe_expert_ffn_q%d (gate/up + down, routed + shared)" % wl.fmt),
                      "achieved": achieved, "peak": hbm_peak, "peak_kind": peak_kind, "unit": "GB/s",
                      "frac": achieved / hbm_peak, "traffic": _profiled_traffic(wl.name) if fused else None,
                      "bytes_per_launch": kern_bytes,
                      "avg_launch_us": ffn_avg_s * 1e6}),
        "e2e": {"value": replicas.job_throughput(T * args.steps, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": L * T * wl.d * 2, "d2h_bytes_per_step": L * T * wl.d * 4},
        "clocks": clocks, "gpu_launches": launches_per_step * args.steps, "dev_status": status,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    if host_leg is not None:
        line["host_miss_completion"] = host_leg
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode_T1_d2048_E512_k10_f768_q2")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-host-misses", action="store_true",
                    help="stacked layers: skip timing the host completion of the miss lists")
    ap.add_argument("--clocks-dir", default=None,
                    help="keep the raw nvidia-smi clock samples of the timed region in this directory")
    ap.add_argument("--combine", choices=["atomic", "kernel"], default="kernel",
                    help="steps path: gate-weighted atomics in the routed expert call (atomic) or y_perm + moe_combine")
    ap.add_argument("--path", choices=["auto", "fused", "steps"], default="auto",
                    help="auto: one-launch layer for T <= 8 tokens, step-by-step calls otherwise")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from bit_expert_ffn_fp32_b200.configs import WORKLOADS
    wl = WORKLOADS[args.workload]
    rank = _env_int("RANK", 0)
    world = _env_int("WORLD_SIZE", 1)
    local_rank = _env_int("LOCAL_RANK", 0)
    if args.impl == "reference":
        return run_reference(args, wl, rank)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_ours(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
