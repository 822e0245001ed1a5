"""Time the host completion of misses (moe_complete_misses_host).

    python -m bit_expert_ffn_fp32_b200.host_bench [--experts 8 --tokens-per-expert 1 --threads 1 --reps 3]

Generates --experts seeded experts of the decode shapes (d=2048, f=768) in
canonical host storage, one miss record per (expert, token), and times the
completion of all records; prints one JSON line per format (Q2, Q3) with the
time per record and per expert and thread.
"""
from __future__ import annotations

import argparse
import json
import os
import time

import numpy as np

from . import native, synth

MISS_DTYPE = np.dtype([("layer", "<i4"), ("expert", "<i4"), ("token", "<i4"), ("j", "<i4"), ("gate", "<f4")])


def time_completion(fmt: int, n_experts: int, per_expert: int, threads: int, reps: int, d: int = 2048, f: int = 768):
    canon = {e: synth.gen_expert(0, 0, e, fmt, d, f) for e in range(n_experts)}
    tab = native.expert_table(n_experts, canon)
    T = per_expert
    x = synth.gen_x(0, 0, T, d)
    recs = np.array([(0, e, t, e % 10, 0.1) for e in range(n_experts) for t in range(T)], MISS_DTYPE)
    y = np.zeros((T, d), np.float32)
    native.complete_misses_host(fmt, d, f, tab, n_experts, recs, len(recs), 0, x, T, y, threads)  # warm-up
    t0 = time.perf_counter()
    for _ in range(reps):
        native.complete_misses_host(fmt, d, f, tab, n_experts, recs, len(recs), 0, x, T, y, threads)
    dt = (time.perf_counter() - t0) / reps
    nth = threads if threads > 0 else len(os.sched_getaffinity(0))
    return {"fmt": "q%d" % fmt, "records": len(recs), "experts": n_experts, "threads": nth,
            "ms_per_call": dt * 1e3, "ms_per_record": dt / len(recs) * 1e3,
            "ms_per_expert_per_thread": dt * min(nth, n_experts) / n_experts * 1e3, "d": d, "f": f}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--experts", type=int, default=8)
    ap.add_argument("--tokens-per-expert", type=int, default=1)
    ap.add_argument("--threads", type=int, default=1)
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args()
    for fmt in (2, 3):
        print(json.dumps(time_completion(fmt, a.experts, a.tokens_per_expert, a.threads, a.reps)))


if __name__ == "__main__":
    main()
