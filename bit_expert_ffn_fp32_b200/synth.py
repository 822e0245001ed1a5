"""Seeded synthetic inputs for one sparse-MoE FFN layer.

This module is the single source of inputs for both the CUDA library and the
CPU oracle. It draws numbers and lays them out in the canonical storage
formats; it holds none of the layer's arithmetic (no routing, no dequantising,
no FFN math), so nothing the two sides compute can leak through it.

Canonical storage (what every consumer reads; the library repacks it itself):

* activations ``x``: bf16 bit patterns, ``uint16 [T][d]``, from fp32 N(0,1)
  rounded to nearest-even.
* router ``Wr``: ``float32 [E][d]``, N(0, 1/d) (standard deviation 1/sqrt(d)),
  optional per-expert ``bias`` ``float32 [E]``.
* a quantised matrix ``[R][K]`` (K runs along 64-weight blocks):
  - ``codes``: ``uint8 [R][K/4]``; weight k of a row sits at byte k//4, bits
    2*(k%4)..2*(k%4)+1 (least significant first). For Q2 this is the whole
    code; for Q3 it is the low two bits.
  - ``hi`` (Q3 only): ``uint8 [R][K/8]``; the third code bit of weight k sits
    at byte k//8, bit k%8.
  - ``scale``: fp16 bit patterns ``uint16 [R][K/64]``, |N(0, 0.02)|.
  - ``min`` (Q2 only): fp16 bit patterns ``uint16 [R][K/64]``, N(0, 0.01).
  Codes are uniform because every stored bit is an independent fair coin.
* an expert is three matrices: ``gate`` and ``up`` are ``[f][d]``, ``down`` is
  ``[d][f]``.

Randomness is counter-based: each tensor gets its own Philox stream keyed by
(seed, layer, expert, tensor), so any expert of any layer can be regenerated
alone and in any order.
"""
from __future__ import annotations

import numpy as np

# Tensor ids inside the Philox key.
_T_X, _T_WR, _T_PERM, _T_EXPERT, _T_TRACE = 1, 2, 3, 4, 5
_MAT_ID = {"gate": 0, "up": 1, "down": 2}
_PART_ID = {"codes": 0, "hi": 1, "scale": 2, "min": 3}


def rng_for(seed: int, *key: int) -> np.random.Generator:
    """Philox generator for one tensor, keyed by (seed, *key)."""
    ss = np.random.SeedSequence([int(seed) & 0xFFFFFFFF, *[int(v) & 0xFFFFFFFF for v in key]])
    return np.random.Generator(np.random.Philox(ss))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); return the bit patterns."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = rounded.astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def f32_to_fp16_bits(a: np.ndarray) -> np.ndarray:
    """Round to IEEE fp16 (numpy's nearest-even conversion); return bit patterns."""
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32).astype(np.float16)).view(np.uint16)


def gen_x(seed: int, layer: int, T: int, d: int, stream: int = 0) -> np.ndarray:
    """Activations: bf16 bits [T][d] from N(0,1). ``stream`` separates replicas/steps."""
    r = rng_for(seed, _T_X, layer, stream, T, d)
    return f32_to_bf16_bits(r.standard_normal((T, d), dtype=np.float32))


def gen_router(seed: int, layer: int, E: int, d: int) -> np.ndarray:
    """Router weights: float32 [E][d], N(0, 1/d)."""
    r = rng_for(seed, _T_WR, layer, E, d)
    return (r.standard_normal((E, d), dtype=np.float32) * np.float32(1.0 / np.sqrt(d))).astype(np.float32)


def gen_rank_perm(seed: int, layer: int, E: int) -> np.ndarray:
    """Popularity rank of each expert, a seeded permutation of 1..E (1 = most popular)."""
    r = rng_for(seed, _T_PERM, layer, E)
    return (r.permutation(E) + 1).astype(np.int64)


def zipf_bias(rank: np.ndarray, alpha: float, s: float = 1.1) -> np.ndarray:
    """Per-expert router bias -alpha*s*ln(rank): skews routing frequencies Zipf-like."""
    return (-alpha * s * np.log(rank.astype(np.float64))).astype(np.float32)


def gen_matrix(seed: int, layer: int, expert: int, which: str, fmt: int, R: int, K: int) -> dict:
    """One quantised matrix [R][K] in canonical storage (see module docstring)."""
    if K % 64:
        raise ValueError("K must be a multiple of 64")
    m = _MAT_ID[which]
    key = (_T_EXPERT, layer, expert, m)
    out = {
        "codes": rng_for(seed, *key, _PART_ID["codes"]).integers(0, 256, (R, K // 4), dtype=np.uint8),
        "scale": f32_to_fp16_bits(np.abs(rng_for(seed, *key, _PART_ID["scale"]).normal(0.0, 0.02, (R, K // 64)))),
    }
    if fmt == 2:
        out["min"] = f32_to_fp16_bits(rng_for(seed, *key, _PART_ID["min"]).normal(0.0, 0.01, (R, K // 64)))
        out["hi"] = None
    elif fmt == 3:
        out["hi"] = rng_for(seed, *key, _PART_ID["hi"]).integers(0, 256, (R, K // 8), dtype=np.uint8)
        out["min"] = None
    else:
        raise ValueError("fmt must be 2 or 3")
    return out


def gen_expert(seed: int, layer: int, expert: int, fmt: int, d: int, f: int) -> dict:
    """A SwiGLU expert: gate/up [f][d] and down [d][f], canonical storage."""
    return {
        "gate": gen_matrix(seed, layer, expert, "gate", fmt, f, d),
        "up": gen_matrix(seed, layer, expert, "up", fmt, f, d),
        "down": gen_matrix(seed, layer, expert, "down", fmt, d, f),
    }


def matrix_from_parts(codes, scale, mn=None, hi=None) -> dict:
    """Assemble a canonical matrix dict from hand-made parts (tests, special cases)."""
    return {
        "codes": np.ascontiguousarray(codes, dtype=np.uint8),
        "scale": np.ascontiguousarray(scale, dtype=np.uint16),
        "min": None if mn is None else np.ascontiguousarray(mn, dtype=np.uint16),
        "hi": None if hi is None else np.ascontiguousarray(hi, dtype=np.uint8),
    }


def slot_table_by_rank(rank: np.ndarray, resident: int, first_slot: int) -> np.ndarray:
    """Residency table for one layer: the ``resident`` most popular experts get
    slots ``first_slot + rank - 1``; every other expert is marked -1 (not resident)."""
    slot = np.full(rank.shape[0], -1, dtype=np.int32)
    hot = rank <= resident
    slot[hot] = (first_slot + rank[hot] - 1).astype(np.int32)
    return slot


def gen_routing_trace(seed: int, L: int, E: int, k: int, n_tokens: int, s: float = 1.1, drift_every: int = 0,
                      drift_swaps: int = 0) -> np.ndarray:
    """Synthetic routing of n_tokens tokens through L layers: int32
    [n_tokens][L][k], each row k distinct expert ids (ascending) drawn without
    replacement with probability proportional to rank^-s, where each layer has
    its own seeded rank permutation. Every drift_every tokens (0 = never), each
    layer exchanges the ranks of drift_swaps random expert pairs: popularity
    drifts the way a conversation changes topic."""
    rng = rng_for(seed, _T_TRACE, L, E, k)
    rank = np.stack([rng.permutation(E) + 1 for _ in range(L)])  # rank[l][e] in 1..E
    out = np.empty((n_tokens, L, k), np.int32)
    for t in range(n_tokens):
        if drift_every and t and t % drift_every == 0:
            for l in range(L):
                for _ in range(drift_swaps):
                    a, b = rng.integers(0, E, 2)
                    rank[l, a], rank[l, b] = rank[l, b], rank[l, a]
        # without replacement: the k largest of log p + Gumbel noise
        keys = -s * np.log(rank) + rng.gumbel(size=(L, E))
        out[t] = np.sort(np.argpartition(-keys, k - 1, axis=1)[:, :k], axis=1)
    return out
