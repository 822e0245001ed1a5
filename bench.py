"""Throughput of one sparse-MoE FFN layer on B200 (C ABI, CUDA kernels).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload all|NAME] [--impl ours|reference]

A step is one pass of the whole layer -- router + top-k, permutation, cache
lookup, routed experts, shared expert, combine -- over one batch of T synthetic
tokens, each step on fresh tokens already resident in HBM. The headline line is
one decode token through a layer of d=2048, 512 experts, top-10 + shared,
f=768, Q2 weights, Zipf-skewed routing, all experts resident. With the default
``--workload all`` the same line carries, under ``workloads``, the other
workloads the metric names, each measured the same way: the MTP verify batch
(T=4, Q3), the 8192-token prefill chunk (Q2) and 48 stacked decode layers with
25% of the experts resident.

Timing: CUDA events on the launching stream around every step. Before each
step a 512 MiB write and then a 256 MiB read of other buffers evict the 126 MB
L2 (the read leaves it holding clean lines, so no write-back of the flush lands
in the timed region): every step reads its weights from HBM. The GPU is kept
busy from the warm-up steps into the timed ones (no idle gap in between).
With N > 1 (torchrun), every rank runs an independent replica on its own
tokens (no collective on the data path); the reported time is the max over
ranks.

--impl reference times the CPU oracle (plain C, fp64) on a bounded sample of
the headline workload on all of the host's cores.
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
HEADLINE = "decode_T1_d2048_E512_k10_f768_q2"
NESTED = ("prefill_T8192_d2048_E512_k10_f768_q2", "verify_T4_d2048_E512_k10_f768_q3",
          # wider MTP verify batches (1 token + 1 or 7 drafts) through the same layer
          "verify_T2_d2048_E512_k10_f768_q3", "verify_T8_d2048_E512_k10_f768_q3",
          "stack48_T1_d2048_E512_k10_f768_q2_res25",
          # beyond the metric's own workloads: a 32K prompt in 8192-token chunks,
          # the 3-bit tier at prefill size and a pool holding both tiers
          "prefill_chunks4_T32768_d2048_E512_k10_f768_q2", "prefill_T8192_d2048_E512_k10_f768_q3",
          "prefill_T8192_d2048_E512_k10_f768_mixed_q3top128")
FLUSH_WRITE_BYTES = 512 << 20
FLUSH_READ_BYTES = 256 << 20


def _env_int(name, default):
    v = os.environ.get(name)
    return int(v) if v not in (None, "") else default


# DRAM bytes (read + written) per launch of the roofline kernel(s) of a
# workload, from one ncu capture (dram__bytes_read.sum + dram__bytes_write.sum;
# see profiles/), valid only while the sources it was captured on are unchanged
# (sha256 of the listed csrc files, first 16 hex digits).
_TC_FILES = ("ffn_tc05.cu", "ffn_mma.cu", "common.cuh", "tc05.cuh", "layout.h", "mma_q.cuh")
_TC_DIGEST = "994a7bb37e842b2b"
PROFILED_TRAFFIC: dict[str, tuple[tuple[str, ...], str, float]] = {
    # the expert-FFN launches of one step (gathers, gate/up, down; routed + shared)
    "prefill_T8192_d2048_E512_k10_f768_q2": (_TC_FILES, _TC_DIGEST, 2503245056.0),
    "prefill_T8192_d2048_E512_k10_f768_q3": (_TC_FILES, _TC_DIGEST, 2738534144.0),
    "prefill_T8192_d2048_E512_k10_f768_mixed_q3top128": (_TC_FILES, _TC_DIGEST, 2874947840.0),
    "prefill_chunks4_T32768_d2048_E512_k10_f768_q2": (_TC_FILES, _TC_DIGEST, 10012321792.0),
}


def _source_digest(files) -> str:
    import hashlib

    m = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "bit_expert_ffn_fp32_b200", "csrc", f), "rb") as fh:
            m.update(fh.read())
    return m.hexdigest()[:16]


def _profiled_traffic(workload: str):
    entry = PROFILED_TRAFFIC.get(workload)
    if entry is None:
        return None
    files, digest, nbytes = entry
    return nbytes if _source_digest(files) == digest else None


def _measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while a workload runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, out_dir: str | None = None, tag: str = ""):
        """The raw samples go to <out_dir>/clocks_gpu<i><tag>.csv (default: a temporary directory)."""
        import tempfile

        self.gpu = gpu_index
        self.proc = None
        d = out_dir or tempfile.mkdtemp(prefix="moe_clocks_")
        self.path = os.path.join(d, f"clocks_gpu{gpu_index}{tag}.csv")

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


# ------------------------------------------------------------------ CPU oracle (baseline and reference arm)
_ORC_CTX = {}


def _oracle_worker_init(wl_name):
    sys.path.insert(0, os.path.join(ROOT, "oracle"))
    import oracle as orc
    from bit_expert_ffn_fp32_b200 import synth
    from bit_expert_ffn_fp32_b200.configs import WORKLOADS, ZIPF_ALPHA

    wl = WORKLOADS[wl_name]
    rank = synth.gen_rank_perm(wl.seed, 0, wl.E)
    _ORC_CTX.update(
        orc=orc, wl=wl, Wr=synth.gen_router(wl.seed, 0, wl.E, wl.d),
        bias=synth.zipf_bias(rank, ZIPF_ALPHA) if wl.zipf else None,
        fmt_of=np.array([wl.expert_fmt(int(r)) for r in rank]),
        shared=synth.gen_expert(wl.seed, 0, wl.E, wl.fmt, wl.d, wl.f), synth=synth)


def _oracle_one_token(stream_id):
    """One oracle layer call on one fresh token of the workload (seconds)."""
    c = _ORC_CTX
    wl, synth = c["wl"], c["synth"]
    x = synth.gen_x(wl.seed, 0, 1, wl.d, stream=stream_id)
    get = lambda e: synth.gen_expert(wl.seed, 0, e, int(c["fmt_of"][e]), wl.d, wl.f)  # noqa: E731
    t0 = time.perf_counter()
    c["orc"].layer(x, c["Wr"], c["bias"], get, c["shared"], wl.k, wl.fmt, fmt_of=c["fmt_of"])
    return time.perf_counter() - t0


class OraclePool:
    """The oracle (as it stands: one single-threaded C call per token) on every
    host core at once: a spawn-started process pool, one token per task."""

    def __init__(self, wl_name: str, cores: int | None = None):
        import multiprocessing as mp

        self.cores = min(cores or len(os.sched_getaffinity(0)), 64)
        self.pool = mp.get_context("spawn").Pool(self.cores, initializer=_oracle_worker_init, initargs=(wl_name,))
        self.pool.map(_oracle_one_token, range(900_000, 900_000 + self.cores))  # imports and first calls

    def throughput(self, layers: int, budget_s: float, stream0: int = 30_000):
        """Tokens per second over rounds of one token per core, until budget_s."""
        n, t_start, rounds = 0, time.perf_counter(), 0
        while time.perf_counter() - t_start < budget_s or rounds == 0:
            ids = range(stream0 + n, stream0 + n + self.cores)
            self.pool.map(_oracle_one_token, ids)
            n += self.cores
            rounds += 1
        wall = time.perf_counter() - t_start
        return n / (wall * layers), n, wall

    def close(self):
        self.pool.terminate()
        self.pool.join()


def cpu_baseline_single(wl, budget_s):
    """The oracle single-threaded in this process on a bounded token sample."""
    _oracle_worker_init(wl.name)
    n, t_tot = 0, 0.0
    while t_tot < budget_s and n < 64:
        t_tot += _oracle_one_token(20_000 + n)
        n += 1
    return {"value": n / (t_tot * wl.layers), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} oracle layer calls of 1 token of {wl.name} ({t_tot:.1f} s, single thread, "
                      "dequantisation included" + (f"; x{wl.layers} layers per token" if wl.layers > 1 else "") + ")"}


def cpu_baseline(wl, pool: OraclePool | None, budget_single=8.0, budget_all=8.0):
    single = cpu_baseline_single(wl, budget_single)
    if pool is None:
        return single
    v, n, wall = pool.throughput(wl.layers, budget_all)
    return {"value": v, "unit": "tokens/s", "cores": pool.cores, "kind": "oracle",
            "sample": f"{n} oracle layer calls of 1 token of {wl.name}, one per process on {pool.cores} host "
                      f"cores ({wall:.1f} s wall, dequantisation included"
                      + (f"; x{wl.layers} layers per token" if wl.layers > 1 else "") + ")",
            "single_thread": single}


def run_reference(args, wl, rank):
    if rank != 0:
        return 0
    pool = OraclePool(wl.name)
    try:
        times = []
        for step in range(min(args.warmup, 1) + args.steps):
            t0 = time.perf_counter()
            pool.pool.map(_oracle_one_token, range(40_000 + step * pool.cores, 40_000 + (step + 1) * pool.cores))
            if step >= min(args.warmup, 1):
                times.append(time.perf_counter() - t0)
            if sum(times) > 150.0:
                break
    finally:
        pool.close()
    tot = sum(times) * wl.layers  # a step of a stacked workload is wl.layers layer calls
    value = pool.cores * len(times) / tot
    sample = (f"{len(times)} of {args.steps} steps run (150 s budget); a step is {pool.cores} oracle layer calls "
              f"of 1 token of {wl.name}, one per process on {pool.cores} host cores, dequantisation included"
              + (f"; one layer call per token timed, x{wl.layers} for the {wl.layers} layers" if wl.layers > 1 else ""))
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": wl.name, "tokens_per_step": pool.cores},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": pool.cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ host completion of misses
def _host_miss_leg(stack, wl, x_dev, x_host, reps=3):
    """The stacked layers' misses completed on the host (moe_miss_engine, every
    host thread) for one step's tokens: GPU alone, host alone after the GPU
    (serial), and both overlapped -- the launch writes each layer's miss list
    to mapped pinned memory as the layer ends and the engine starts on it while
    the GPU runs the later layers. Host wall-clock times (the host is the one
    waiting), median of `reps`; the missed experts are generated into host
    storage first (not timed)."""
    import torch

    from bit_expert_ffn_fp32_b200 import native
    from bit_expert_ffn_fp32_b200.layer import MISS_DTYPE

    L, T = wl.layers, wl.T
    sb = stack.stack_buffers(T)
    stack.forward_stack(x_dev, sb)
    torch.cuda.synchronize()
    missed = [sorted(set(m[1] for m in stack.stack_misses(sb, l))) for l in range(L)]
    tabs = [native.expert_table(wl.E, {e: stack.canonical_expert(l, e) for e in missed[l]}) for l in range(L)]
    hb = stack.stack_buffers(T, host_misses=True)
    cap = hb.idx.shape[1]
    cnt = hb.miss_count.view(np.int32)
    miss_h = hb.miss.view(MISS_DTYPE, (L, cap))
    xs = [np.ascontiguousarray(x_host[l]) for l in range(L)]
    y_add = np.zeros((L, T, wl.d), np.float32)
    threads = len(os.sched_getaffinity(0))
    eng = native.MissEngine(0)
    gpu, host, both = [], [], []
    try:
        for _ in range(reps):
            cnt[:] = -1
            t0 = time.perf_counter()
            stack.forward_stack(x_dev, hb)
            torch.cuda.synchronize()
            gpu.append(time.perf_counter() - t0)
            y_add[:] = 0
            t0 = time.perf_counter()
            for l in range(L):
                eng.submit(wl.fmt, wl.d, wl.f, tabs[l], wl.E, miss_h[l], cnt[l:l + 1], cap, l, xs[l], T, y_add[l])
            eng.wait()
            host.append(time.perf_counter() - t0)
            cnt[:] = -1
            y_add[:] = 0
            t0 = time.perf_counter()
            stack.forward_stack(x_dev, hb)
            for l in range(L):
                eng.submit(wl.fmt, wl.d, wl.f, tabs[l], wl.E, miss_h[l], cnt[l:l + 1], cap, l, xs[l], T, y_add[l])
            eng.wait()
            torch.cuda.synchronize()
            both.append(time.perf_counter() - t0)
    finally:
        eng.close()
    n_rec = int(sum(int(c) for c in cnt))
    g, h, o = (1e3 * float(np.median(v)) for v in (gpu, host, both))
    return {"gpu_ms": g, "host_ms": h, "serial_ms": g + h, "overlapped_ms": o,
            "tokens_per_s_overlapped": T / (o / 1e3), "misses_per_step": n_rec,
            "distinct_experts_per_step": int(sum(len(m) for m in missed)), "threads": threads,
            "call": "moe_stack_decode writing miss lists to mapped host memory + moe_miss_engine (host C++ workers, "
                    "fp32 dot products on the canonical codes)",
            "timing": f"host wall clock, median of {reps}; serial = GPU alone + host alone"}


# ------------------------------------------------------------------ our arm
class Evictor:
    """Leaves the L2 holding none of the workload's bytes and no dirty lines."""

    def __init__(self, torch, dev):
        self.torch = torch
        self.w = torch.empty(FLUSH_WRITE_BYTES // 4, dtype=torch.float32, device=dev)
        self.r = torch.ones(FLUSH_READ_BYTES // 4, dtype=torch.float32, device=dev)
        self.out = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self, i):
        self.w.fill_(float(i))
        self.torch.sum(self.r, 0, out=self.out)


def measure(wl, stack, args, rank, world, local_rank, dev, evict):
    """One workload: warm-up, timed steps, kernel-only timing, routing
    statistics and the end-to-end pass; returns the fields of its JSON line."""
    import torch

    from bit_expert_ffn_fp32_b200 import native, replicas, synth
    from bit_expert_ffn_fp32_b200.layer import x_tensor

    L, T = wl.layers, wl.T
    stream = torch.cuda.current_stream()
    steps, warmup = args.steps, args.warmup
    n_steps = warmup + steps
    # steps get their own tokens, generated up front and resident in HBM (at most
    # 256 MiB of distinct inputs, cycled; the L2 is evicted between steps anyway)
    n_x = max(1, min(n_steps, (256 << 20) // (L * T * wl.d * 2)))
    xs_host = [np.stack([synth.gen_x(wl.seed, l, T, wl.d, stream=s) for l in range(L)])
               for s in replicas.token_streams(rank, n_x)]
    xs_dev = torch.stack([torch.stack([x_tensor(xl, dev) for xl in x]) for x in xs_host])
    xs = lambda i: xs_dev[i % n_x]  # noqa: E731

    fused = T <= 8 and not stack.mixed
    stacked = fused and L > 1  # all layers in one moe_stack_decode launch
    sb = stack.stack_buffers(T) if stacked else None
    C = wl.chunk if wl.chunk and not fused else T   # tokens per forward() (a prompt's chunks)
    chunks = [(c0, min(C, T - c0)) for c0 in range(0, T, C)]
    y_long = torch.empty((T, wl.d), dtype=torch.float32, device=dev) if len(chunks) > 1 else None
    b = stack.buffers(T) if y_long is None else None

    def layer_step(xset, evs=None):
        """One step; evs: one event pair per chunk, recorded around the expert
        calls (or the whole launch on the one-launch paths). Returns y."""
        if fused:
            if evs:
                evs[0][0].record(stream)
            if stacked:
                stack.forward_stack(xset, sb)
            else:
                stack.forward_fused(0, xset[0], b)
            if evs:
                evs[0][1].record(stream)
            return sb.y if stacked else b.y
        if y_long is not None:
            return stack.forward_chunked(0, xset[0], C, y=y_long, ffn_events=evs)
        stack.forward(0, xset[0], b, ffn_events=evs[0] if evs else None)
        return b.y

    tc_path = not fused and C * wl.k >= 512
    launches_per_step = 1 if fused else sum(stack.launches(n) for _, n in chunks)
    statuses = [sb.status] if stacked else [stack.buffers(n).status for n in sorted({n for _, n in chunks})]

    for st in statuses:
        st.zero_()
    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    ev = [(mk(), mk()) for _ in range(steps)]
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank, args.clocks_dir, tag="_" + wl.name)
    sampler.start()
    # warm-up steps straight into the timed ones: the GPU never idles in between
    for s in range(warmup):
        evict(s)
        layer_step(xs(s))
    for i in range(steps):
        evict(i)
        ev[i][0].record(stream)
        layer_step(xs(warmup + i))
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    step_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(steps)]
    total_ms = sum(step_ms)
    # The dominant kernel's own time, for the roofline line: the same steps again
    # with events around it (kept out of the timed steps above, whose value they
    # would inflate). With one launch per layer it is the step itself.
    if fused:
        kern_ms = step_ms
    else:
        kev = [[(mk(), mk()) for _ in chunks] for _ in range(steps)]
        for i in range(steps):
            evict(i)
            layer_step(xs(warmup + i), kev[i])
        torch.cuda.synchronize()
        kern_ms = [sum(a.elapsed_time(c) for a, c in kev[i]) for i in range(steps)]
    status = 0
    for st in statuses:
        status |= int(st.item())

    # distinct resident experts (and their packed bytes), resident pairs and
    # misses of each step's routing, summed over the layers and the chunks (not timed)
    ebytes = [np.array([native.expert_bytes(stack.expert_fmt(l, e), wl.d, wl.f) for e in range(wl.E)])
              for l in range(L)]
    n_act, n_bytes, n_pairs, n_miss = [], [], [], []
    for i in range(min(steps, (64 if T <= 64 else 4) if L == 1 else 4)):
        a_sum = p_sum = m_sum = by_sum = 0
        if stacked:
            layer_step(xs(warmup + i))
            idx_h = sb.idx[:, : T * wl.k].cpu().numpy()
            sop_h = sb.sop[:, : T * wl.k].cpu().numpy()
            mc_h = sb.miss_count.cpu().numpy()
            for l in range(L):
                ids = np.unique(idx_h[l])
                ids = ids[stack.slot_of_host[l][ids] >= 0]
                a_sum += len(ids)
                by_sum += int(ebytes[l][ids].sum())
                p_sum += int((sop_h[l] >= 0).sum())
                m_sum += int(mc_h[l])
        else:
            x0 = xs(warmup + i)[0]
            for c0, n in chunks:
                bl = stack.buffers(n)
                if fused:
                    stack.forward_fused(0, x0, bl)
                else:
                    stack.forward(0, x0[c0:c0 + n], bl)
                na = int(bl.active[0].item())
                ids = bl.active[1:1 + na].cpu().numpy()
                ids = ids[stack.slot_of_host[0][ids] >= 0]
                a_sum += len(ids)
                by_sum += int(ebytes[0][ids].sum())
                p_sum += int((bl.sop[: n * wl.k] >= 0).sum().item())
                m_sum += int(bl.miss_count.item())
        n_act.append(a_sum)
        n_bytes.append(by_sum)
        n_pairs.append(p_sum)
        n_miss.append(m_sum)
    mean_act = float(np.mean(n_act))
    res_pairs_mean = float(np.mean(n_pairs))
    hit_rate = res_pairs_mean / (L * T * wl.k)

    # ---- e2e: pinned host tokens in, layer, result out, every step
    x_pin = torch.from_numpy(np.stack(xs_host).view(np.int16)).pin_memory()  # [n_x][L][T][d]
    n_y = min(steps, max(2, (256 << 20) // (L * T * wl.d * 4)))
    y_pin = torch.empty((n_y, L, T, wl.d), dtype=torch.float32).pin_memory()
    x_dev = torch.empty((L, T, wl.d), dtype=torch.int16, device=dev)
    e2e_ev = [(mk(), mk()) for _ in range(steps)]
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    for i in range(steps):
        evict(i)
        e2e_ev[i][0].record(stream)
        if y_long is not None:  # a chunked prompt: copies of chunks c+1 and c-1 overlap chunk c
            stack.forward_chunked_host(0, x_pin[i % n_x][0], y_pin[i % n_y, 0], C)
        else:
            x_dev.copy_(x_pin[i % n_x], non_blocking=True)
            y_out = layer_step(x_dev)
            if stacked:
                y_pin[i % n_y].copy_(y_out[:, :T], non_blocking=True)
            else:
                y_pin[i % n_y, 0].copy_(y_out[:T], non_blocking=True)
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    e2e_ms = sum(e2e_ev[i][0].elapsed_time(e2e_ev[i][1]) for i in range(steps))
    total_ms, kern_total, e2e_ms = replicas.max_over_ranks([total_ms, sum(kern_ms), e2e_ms], device=dev)

    hbm_peak, tc_peak, peak_kind = _measured_peaks()
    eb = native.expert_bytes(wl.fmt, wl.d, wl.f)
    # routed resident experts (each in its own format) + the shared experts, read once
    ffn_bytes = float(np.mean(n_bytes)) + L * eb
    layer_bytes = L * wl.E * wl.d * 4 + ffn_bytes  # + the fp32 router weights (all L layers of a step)
    kern_avg_s = kern_total / steps / 1e3
    ffn_flops = 2.0 * 3 * wl.d * wl.f * (res_pairs_mean + T)   # routed resident pairs + shared, per step
    traffic = _profiled_traffic(wl.name)
    fmt_names = "/".join("q%d" % fm for fm in stack.fmts)
    if tc_path and not fused:
        roof = {"bound": "tensor",
                "kernel": "moe_expert_ffn_%s tcgen05 grouped GEMMs (gate/up + down, routed + shared%s)"
                          % (fmt_names, ", every chunk" if len(chunks) > 1 else ""),
                "achieved": ffn_flops / kern_avg_s / 1e12, "peak": tc_peak, "peak_kind": peak_kind + " bf16 burst",
                "unit": "TFLOP/s", "frac": ffn_flops / kern_avg_s / 1e12 / tc_peak, "traffic": traffic,
                "traffic_scope": "the expert FFN launches of one step (fp16 gathers, gate/up, down; routed + shared)",
                "flops_per_launch": ffn_flops, "avg_launch_us": kern_avg_s * 1e6}
    else:
        kb = layer_bytes if fused else ffn_bytes
        roof = {"bound": "hbm",
                "kernel": ("decode_layer_kernel (moe_stack_decode: %d layers in one launch)" % L if stacked else
                           "decode_layer_kernel (moe_layer_decode: whole layer, one launch)") if fused else
                          "moe_expert_ffn_%s (gate/up + down, routed + shared)" % fmt_names,
                "achieved": kb / kern_avg_s / 1e9, "peak": hbm_peak, "peak_kind": peak_kind, "unit": "GB/s",
                "frac": kb / kern_avg_s / 1e9 / hbm_peak, "traffic": traffic,
                "traffic_scope": "DRAM bytes per step (all launches of the step)",
                "traffic_note": None if traffic is not None else
                ("no ncu capture: its kernel replay of the cooperative cluster launch failed to launch; "
                 "the phase trace build times the kernel instead" if fused else
                 "no ncu capture of these sources"),
                "bytes_per_launch": kb, "avg_launch_us": kern_avg_s * 1e6}
    line = {
        "value": replicas.job_throughput(T * steps, world, total_ms), "unit": "tokens/s",
        "ms_per_step": total_ms / steps,
        "step_ms_quantiles": {"median": float(np.median(step_ms)), "p90": float(np.percentile(step_ms, 90)),
                              "min": float(np.min(step_ms)), "max": float(np.max(step_ms)),
                              "note": "this rank's per-step CUDA-event times"},
        "dtype": ("f16 (dequantised %s) x f16 -> f32" % fmt_names if tc_path and not fused
                  else "%sxf16->f32" % fmt_names),
        "config": {"workload": wl.name, "tokens_per_step": T,
                   "l2": "512 MiB write + 256 MiB read of other buffers between steps (flushed, clean)",
                   "path": ("moe_stack_decode (all layers, one launch)" if stacked else
                            "moe_layer_decode (one launch)") if fused else
                           ("step-by-step calls, y_perm + moe_combine"
                            + (", %d chunks of <= %d tokens back to back" % (len(chunks), C) if len(chunks) > 1
                               else "")
                            + (", one expert call per format (mixed pool)" if stack.mixed else "")),
                   "parallelism": f"replicas x{world}", "layers_per_step": L,
                   "step_algorithmic_bytes": layer_bytes,
                   "step_GBps": layer_bytes / (total_ms / steps / 1e3) / 1e9,
                   "mean_distinct_resident_experts": mean_act, "hit_rate": hit_rate,
                   "misses_per_step": float(np.mean(n_miss))},
        "roofline": roof,
        "e2e": {"value": replicas.job_throughput(T * steps, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": L * T * wl.d * 2, "d2h_bytes_per_step": L * T * wl.d * 4,
                "path": ("MoEStack.forward_chunked_host: chunk copies in and out on two side streams, "
                         "overlapped with the neighbouring chunks' layers" if y_long is not None else
                         "pinned x copied in, the step, y copied out, on one stream")},
        "clocks": clocks, "gpu_launches": launches_per_step * steps, "dev_status": status,
    }
    if stacked and not args.no_host_misses and rank == 0:
        i_last = (warmup + steps - 1) % n_x
        line["host_miss_completion"] = _host_miss_leg(stack, wl, xs(warmup + steps - 1), xs_host[i_last])
    return line


def run_ours(args, names, rank, world, local_rank):
    import torch

    from bit_expert_ffn_fp32_b200.configs import WORKLOADS
    from bit_expert_ffn_fp32_b200.layer import MoEStack

    want_cpu = world == 1 and not args.no_cpu_baseline
    pool = OraclePool(names[0]) if want_cpu else None  # spawn-started, before any GPU work
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    evict = Evictor(torch, dev)
    stacks = {}
    lines = {}
    try:
        for name in names:
            wl = WORKLOADS[name]
            # workloads that differ only in T share one pool of experts
            key = (wl.d, wl.E, wl.f, wl.fmt, wl.layers, wl.resident, wl.seed, wl.zipf, wl.q3_top)
            if key not in stacks:
                stacks.clear()
                torch.cuda.empty_cache()
                stacks[key] = MoEStack(wl, device=dev)
            lines[name] = measure(wl, stacks[key], args, rank, world, local_rank, dev, evict)
            if want_cpu and rank == 0:
                if name == names[0]:
                    lines[name]["cpu_baseline"] = cpu_baseline(wl, pool, 8.0, 10.0)
                else:
                    lines[name]["cpu_baseline"] = cpu_baseline(wl, None, 5.0)
    finally:
        if pool is not None:
            pool.close()
    if rank != 0:
        return 0
    head = lines[names[0]]
    line = {"metric": METRIC, "value": head.pop("value"), "unit": head.pop("unit"), "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head.pop("ms_per_step"),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "data": "synthetic"}
    line.update(head)
    if len(names) > 1:
        line["workloads"] = {n: lines[n] for n in names[1:]}
        line["gpu_launches"] = sum(lines[n]["gpu_launches"] for n in names)
        line["gpu_launches_note"] = "all workloads of this run (headline: %d)" % head["gpu_launches"]
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="all", help="all (headline + nested workloads) or one workload name")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-host-misses", action="store_true",
                    help="stacked layers: skip timing the host completion of the miss lists")
    ap.add_argument("--clocks-dir", default=None,
                    help="keep the raw nvidia-smi clock samples of each workload in this directory")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from bit_expert_ffn_fp32_b200.configs import WORKLOADS
    names = [HEADLINE, *NESTED] if args.workload == "all" else [args.workload]
    for n in names:
        if n not in WORKLOADS:
            ap.error(f"unknown workload {n}")
    rank = _env_int("RANK", 0)
    world = _env_int("WORLD_SIZE", 1)
    local_rank = _env_int("LOCAL_RANK", 0)
    if args.impl == "reference":
        return run_reference(args, WORKLOADS[names[0]], rank)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_ours(args, names, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
