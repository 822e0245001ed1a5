"""Python face of the CPU oracle -- TEST INFRASTRUCTURE ONLY.

Wraps oracle/moe_oracle.c (plain C, fp64 apart from the fp32 router logit) and
assembles one MoE FFN layer from its steps. Only tests, the package smoke check
and bench.py's CPU-baseline leg may import this module; the CUDA library never
does, and this module never imports the library.

Layer definition (per token t):
  1. router logits l[t][e] (fp32, fixed operation order, see moe_oracle.c);
  2. the top-k experts by (logit desc, id asc), reported in ascending id, with
     gates = softmax over the k selected logits (fp64);
  3. the stable permutation of the T*k (token, slot) pairs by expert;
  4. the cache lookup: pairs whose expert has no HBM slot are misses;
  5. y_partial[t] = FFN_shared(x_t) + sum over resident selected experts of
     gate * FFN_e(x_t); y_full adds the missed experts too.
FFN_e is the SwiGLU expert on dequantised fp64 weights; every expert is
dequantised by its own storage format (the layer's, or fmt_of[e] for a pool
holding both tiers).
"""
from __future__ import annotations

import ctypes as C
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import build_oracle  # noqa: E402

_P = C.c_void_p


class _Miss(C.Structure):
    _fields_ = [("layer", C.c_int32), ("expert", C.c_int32), ("token", C.c_int32),
                ("j", C.c_int32), ("gate", C.c_float)]


def _load():
    lib = C.CDLL(build_oracle.build())
    lib.orc_bf16_value.restype = C.c_double
    lib.orc_bf16_value.argtypes = [C.c_uint16]
    lib.orc_fp16_value.restype = C.c_double
    lib.orc_fp16_value.argtypes = [C.c_uint16]
    lib.orc_dequant_q2.argtypes = [_P, _P, _P, C.c_int, C.c_int, _P]
    lib.orc_dequant_q3.argtypes = [_P, _P, _P, C.c_int, C.c_int, _P]
    lib.orc_router_logit.restype = C.c_float
    lib.orc_router_logit.argtypes = [_P, _P, C.c_int, _P]
    lib.orc_router.argtypes = [_P, _P, _P, C.c_int, C.c_int, C.c_int, _P, _P, _P]
    lib.orc_topk.restype = C.c_int
    lib.orc_topk.argtypes = [_P, C.c_int, C.c_int, C.c_int, _P, _P]
    lib.orc_permute.restype = C.c_int
    lib.orc_permute.argtypes = [_P, C.c_int, C.c_int, C.c_int, _P, _P, _P, _P, _P, _P]
    lib.orc_cache_lookup.restype = C.c_int
    lib.orc_cache_lookup.argtypes = [_P, C.c_int, _P, _P, C.c_int, C.c_int, C.c_int, _P, _P, C.c_int]
    lib.orc_expert_ffn.argtypes = [_P, _P, _P, _P, C.c_int, C.c_int, _P, _P]
    lib.orc_expert_ffn_batch.argtypes = [_P, _P, _P, _P, C.c_int, C.c_int, C.c_int, _P]
    return lib


_lib = _load()


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_P)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- formats
def bf16_value(bits: int) -> float:
    return _lib.orc_bf16_value(int(bits))


def fp16_value(bits: int) -> float:
    return _lib.orc_fp16_value(int(bits))


def bf16_to_f64(x_bits: np.ndarray) -> np.ndarray:
    """Activations from bf16 bits to fp64 (exact)."""
    u = _c(x_bits, np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def dequant(mat: dict, fmt: int) -> np.ndarray:
    """fp64 weights [R][K] of one canonical quantised matrix."""
    codes = _c(mat["codes"], np.uint8)
    R, K = codes.shape[0], codes.shape[1] * 4
    W = np.empty((R, K), dtype=np.float64)
    scale = _c(mat["scale"], np.uint16)
    if fmt == 2:
        _lib.orc_dequant_q2(_ptr(codes), _ptr(scale), _ptr(_c(mat["min"], np.uint16)), R, K, _ptr(W))
    elif fmt == 3:
        _lib.orc_dequant_q3(_ptr(codes), _ptr(_c(mat["hi"], np.uint8)), _ptr(scale), R, K, _ptr(W))
    else:
        raise ValueError("fmt")
    return W


def dequant_expert(expert: dict, fmt: int) -> dict:
    return {m: dequant(expert[m], fmt) for m in ("gate", "up", "down")}


# ---------------------------------------------------------------- router
def router_logit(x_row: np.ndarray, w_row: np.ndarray, bias: float | None = None) -> np.float32:
    x_row = _c(x_row, np.uint16)
    w_row = _c(w_row, np.float32)
    b = None if bias is None else np.array([bias], dtype=np.float32)
    return np.float32(_lib.orc_router_logit(_ptr(x_row), _ptr(w_row), x_row.shape[0], _ptr(b)))


def router(x: np.ndarray, Wr: np.ndarray, bias: np.ndarray | None):
    """(logit32 [T][E] fp32, logit64 [T][E], absdot [T][E])."""
    x = _c(x, np.uint16)
    Wr = _c(Wr, np.float32)
    T, d = x.shape
    E = Wr.shape[0]
    b = None if bias is None else _c(bias, np.float32)
    l32 = np.empty((T, E), np.float32)
    l64 = np.empty((T, E), np.float64)
    ad = np.empty((T, E), np.float64)
    _lib.orc_router(_ptr(x), _ptr(Wr), _ptr(b), T, d, E, _ptr(l32), _ptr(l64), _ptr(ad))
    return l32, l64, ad


def logit_error_bound(d: int, absdot: np.ndarray, bias: np.ndarray | None) -> np.ndarray:
    """Bound on |fp32 contract logit - exact logit|: a chain of d/32 fused
    multiply-adds, five pairwise additions and the bias addition, each with unit
    roundoff u = 2^-24 (gamma_n = n u / (1 - n u)), plus the fp64 reference's own
    error."""
    u = 2.0 ** -24
    n = d // 32 + 6
    g = n * u / (1 - n * u)
    b = 0.0 if bias is None else np.abs(np.asarray(bias, np.float64))[None, :]
    u64 = 2.0 ** -53
    return g * (absdot + b) + d * u64 / (1 - d * u64) * absdot


def topk(logits: np.ndarray, k: int):
    """(idx int32 [T][k] ascending ids, gate fp64 [T][k])."""
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    gate = np.empty((T, k), np.float64)
    if _lib.orc_topk(_ptr(logits), T, E, k, _ptr(idx), _ptr(gate)) != 0:
        raise ValueError("non-finite router logit")
    return idx, gate


# ---------------------------------------------------------------- permutation / cache
def permute(idx: np.ndarray, E: int) -> dict:
    idx = _c(idx, np.int32)
    T, k = idx.shape
    n = T * k
    out = {
        "counts": np.empty(E, np.int32), "offsets": np.empty(E + 1, np.int32),
        "sorted_tok": np.empty(n, np.int32), "sorted_j": np.empty(n, np.int32),
        "inv": np.empty(n, np.int32), "active": np.zeros(E + 1, np.int32),
    }
    rc = _lib.orc_permute(_ptr(idx), T, k, E, *(_ptr(out[key]) for key in
                                                 ("counts", "offsets", "sorted_tok", "sorted_j", "inv", "active")))
    if rc != 0:
        raise ValueError("expert id out of range")
    return out


def cache_lookup(slot_of: np.ndarray, layer: int, idx: np.ndarray, gate: np.ndarray, E: int,
                 miss_cap: int | None = None):
    """(slot_of_pair int32 [T*k], misses list of (layer, expert, token, j, gate), miss count)."""
    slot_of = _c(slot_of, np.int32)
    idx = _c(idx, np.int32)
    gate = _c(gate, np.float64)
    T, k = idx.shape
    cap = T * k if miss_cap is None else miss_cap
    sop = np.empty(T * k, np.int32)
    miss = (_Miss * max(cap, 1))()
    n = _lib.orc_cache_lookup(_ptr(slot_of), layer, _ptr(idx), _ptr(gate), T, k, E, _ptr(sop),
                              C.cast(miss, _P), cap)
    recs = [(m.layer, m.expert, m.token, m.j, m.gate) for m in miss[:min(n, cap)]]
    return sop, recs, n


# ---------------------------------------------------------------- experts
def expert_ffn(W: dict, x: np.ndarray) -> np.ndarray:
    """SwiGLU expert on fp64 weights; x is fp64 [n][d]; returns fp64 [n][d]."""
    x = _c(np.atleast_2d(x), np.float64)
    n, d = x.shape
    f = W["gate"].shape[0]
    y = np.empty((n, d), np.float64)
    _lib.orc_expert_ffn_batch(_ptr(_c(W["gate"], np.float64)), _ptr(_c(W["up"], np.float64)),
                              _ptr(_c(W["down"], np.float64)), _ptr(x), n, d, f, _ptr(y))
    return y


def expert_hidden(W: dict, x_row: np.ndarray) -> np.ndarray:
    """h = silu(Wg x) * (Wu x) for one token (fp64 [f])."""
    x_row = _c(x_row, np.float64)
    d = x_row.shape[0]
    f = W["gate"].shape[0]
    y = np.empty(d, np.float64)
    h = np.empty(f, np.float64)
    _lib.orc_expert_ffn(_ptr(_c(W["gate"], np.float64)), _ptr(_c(W["up"], np.float64)),
                        _ptr(_c(W["down"], np.float64)), _ptr(x_row), d, f, _ptr(y), _ptr(h))
    return h


def layer(x: np.ndarray, Wr: np.ndarray, bias, get_expert, shared: dict, k: int, fmt: int,
          slot_of: np.ndarray | None = None, layer_id: int = 0, tokens=None, miss_cap=None,
          fmt_of=None) -> dict:
    """One MoE FFN layer.

    get_expert(e) returns expert e in canonical storage; shared is the shared
    expert. slot_of (int32 [E], -1 = not resident) defaults to all resident.
    fmt is the storage format of every expert, unless fmt_of (int [E]) gives
    each routed expert its own (a pool holding both tiers: each expert is
    dequantised by its own format's rule, the shared expert by fmt).
    tokens restricts the FFN work to those token indices (routing, permutation
    and lookup always cover all T tokens); y_partial / y_full rows of other
    tokens are NaN.
    """
    x = _c(x, np.uint16)
    T, d = x.shape
    E = Wr.shape[0]
    l32, l64, ad = router(x, Wr, bias)
    idx, gate = topk(l32, k)
    perm = permute(idx, E)
    if slot_of is None:
        slot_of = np.arange(E, dtype=np.int32)
    sop, misses, nmiss = cache_lookup(slot_of, layer_id, idx, gate, E, miss_cap)
    toks = list(range(T)) if tokens is None else list(tokens)
    xf = bf16_to_f64(x)
    y_part = np.full((T, d), np.nan)
    y_full = np.full((T, d), np.nan)
    # Every needed FFN_e(x_t) is evaluated once, one expert at a time (so that
    # only one expert's fp64 matrices are held at once); the per-token sums
    # below then add them in the definition's order.
    ffn: dict[tuple[int, int], np.ndarray] = {}
    need: dict[int, list[int]] = {}
    for t in toks:
        for j in range(k):
            need.setdefault(int(idx[t, j]), []).append(t)
    for e in sorted(need):
        W = dequant_expert(get_expert(e), fmt if fmt_of is None else int(fmt_of[e]))
        ts = sorted(set(need[e]))
        rows = expert_ffn(W, xf[ts])
        for i, t in enumerate(ts):
            ffn[(e, t)] = rows[i]
        del W
    Wsh = dequant_expert(shared, fmt)
    for t in toks:
        acc_hit = expert_ffn(Wsh, xf[t])[0]
        acc_all = acc_hit.copy()
        for j in range(k):
            e = int(idx[t, j])
            ye = gate[t, j] * ffn[(e, t)]
            acc_all = acc_all + ye
            if slot_of[e] >= 0:
                acc_hit = acc_hit + ye
        y_part[t] = acc_hit
        y_full[t] = acc_all
    return {"logit32": l32, "logit64": l64, "absdot": ad, "idx": idx, "gate": gate, "perm": perm,
            "slot_of_pair": sop, "misses": misses, "miss_count": nmiss,
            "y_partial": y_part, "y_full": y_full, "tokens": list(toks)}
