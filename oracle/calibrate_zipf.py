"""Re-derive ZIPF_ALPHA (bit_expert_ffn_fp32_b200/configs.py) -- test infrastructure.

The router bias -alpha * 1.1 * ln(rank) skews expert popularity Zipf-like. alpha
is found by bisection so that, over a chunk of tokens, the most popular expert
is selected by about 2000/8192 of the tokens (per-expert counts then range from
0 to about 2000 in an 8192-token prefill chunk). Uses the oracle's router and
top-k only. Run: python oracle/calibrate_zipf.py [tokens]
"""
from __future__ import annotations

import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import oracle  # noqa: E402
from bit_expert_ffn_fp32_b200 import synth  # noqa: E402


def top_share(l0: np.ndarray, rank: np.ndarray, alpha: float, k: int) -> float:
    logits = (l0 + synth.zipf_bias(rank, alpha)[None, :]).astype(np.float32)
    idx, _ = oracle.topk(logits, k)
    return np.bincount(idx.ravel(), minlength=l0.shape[1]).max() / l0.shape[0]


def main(T: int = 1024, d: int = 2048, E: int = 512, k: int = 10, target: float = 2000 / 8192):
    x = synth.gen_x(7, 0, T, d)
    Wr = synth.gen_router(7, 0, E, d)
    rank = synth.gen_rank_perm(7, 0, E)
    l0, _, _ = oracle.router(x, Wr, None)
    lo, hi = 0.0, 2.0
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        if top_share(l0, rank, mid, k) < target:
            lo = mid
        else:
            hi = mid
    print(f"alpha = {0.5 * (lo + hi):.4f}  (top share {top_share(l0, rank, 0.5 * (lo + hi), k):.4f})")


if __name__ == "__main__":
    main(int(sys.argv[1]) if len(sys.argv) > 1 else 1024)
