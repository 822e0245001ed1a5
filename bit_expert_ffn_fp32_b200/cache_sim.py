"""Hit rate of the expert-cache policy on a synthetic routing trace.

    python -m bit_expert_ffn_fp32_b200.cache_sim [--layers 48 --experts 512 --slots 6144 --tokens 4000]

Routing follows Zipf(s) popularity per layer with a drift (random rank
exchanges every --drift-every tokens). Compared on the same trace: the online
policy (moe_cache_policy_*: counts halved every --epoch tokens, a plan every
--plan-every tokens with at most --max-swaps changes), and a resident set fixed
from the counts of the first --warm tokens. Prints one JSON line with both hit
rates and the policy's host cost per observe and per plan.
"""
from __future__ import annotations

import argparse
import json
import time

import numpy as np

from . import native, synth


def simulate(L, E, S, k, tokens, s, drift_every, drift_swaps, epoch, margin, plan_every, max_swaps, warm, seed=0):
    trace = synth.gen_routing_trace(seed, L, E, k, tokens, s=s, drift_every=drift_every, drift_swaps=drift_swaps)
    pol = native.CachePolicy(L, E, S, epoch, margin)
    slot = np.full((L, E), -1, np.int32)
    hits = total = swaps = 0
    t_obs = t_plan = 0.0
    n_plan = 0
    for t in range(tokens):
        for l in range(L):
            row = trace[t, l]
            hits += int((slot[l][row] >= 0).sum())
            total += k
            t0 = time.perf_counter()
            pol.observe(l, row[None, :])
            t_obs += time.perf_counter() - t0
        if (t + 1) % plan_every == 0:
            t0 = time.perf_counter()
            swaps += len(pol.plan(slot, max_swaps))
            t_plan += time.perf_counter() - t0
            n_plan += 1
    cnt = np.stack([np.bincount(trace[:warm, l].ravel(), minlength=E) for l in range(L)]).ravel()
    fixed = np.zeros(L * E, bool)
    fixed[sorted(range(L * E), key=lambda i: (-cnt[i], i))[:S]] = True
    fixed = fixed.reshape(L, E)
    fixed_hits = sum(int(fixed[l][trace[t, l]].sum()) for t in range(tokens) for l in range(L))
    return {"online_hit_rate": hits / total, "fixed_hit_rate": fixed_hits / total, "swaps": swaps,
            "us_per_observe": t_obs / (tokens * L) * 1e6, "ms_per_plan": t_plan / max(n_plan, 1) * 1e3,
            "config": {"layers": L, "experts": E, "slots": S, "k": k, "tokens": tokens, "zipf_s": s,
                       "drift_every": drift_every, "drift_swaps": drift_swaps, "epoch": epoch, "margin": margin,
                       "plan_every": plan_every, "max_swaps": max_swaps, "fixed_from_first": warm}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--layers", type=int, default=48)
    ap.add_argument("--experts", type=int, default=512)
    ap.add_argument("--slots", type=int, default=6144)
    ap.add_argument("--k", type=int, default=10)
    ap.add_argument("--tokens", type=int, default=4000)
    ap.add_argument("--zipf", type=float, default=1.1)
    ap.add_argument("--drift-every", type=int, default=200)
    ap.add_argument("--drift-swaps", type=int, default=64)
    ap.add_argument("--epoch", type=int, default=256)
    ap.add_argument("--margin", type=int, default=1)
    ap.add_argument("--plan-every", type=int, default=16)
    ap.add_argument("--max-swaps", type=int, default=64)
    ap.add_argument("--warm", type=int, default=200)
    a = ap.parse_args()
    print(json.dumps(simulate(a.layers, a.experts, a.slots, a.k, a.tokens, a.zipf, a.drift_every, a.drift_swaps,
                              a.epoch, a.margin, a.plan_every, a.max_swaps, a.warm)))


if __name__ == "__main__":
    main()
