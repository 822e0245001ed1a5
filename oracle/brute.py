"""Pure-Python brute force for tiny layers -- TEST INFRASTRUCTURE ONLY.

An independent second statement of the layer, written the slow way so that
it can pin the C oracle on tiny shapes (T <= 3, d = 128, E <= 8, f = 64):

* fp32 arithmetic is done exactly with fractions and rounded once to the
  nearest binary32 (ties to even), so a fused multiply-add really rounds once;
* top-k enumerates every k-subset and keeps the one with the largest exact
  logit sum, ties going to the lexicographically smallest id tuple;
* the permutation is Python's sorted() on (expert, pair index);
* dequantisation reads one bit at a time; the FFN is triple loops on floats.
"""
from __future__ import annotations

import itertools
import math
import struct
from fractions import Fraction


# ------------------------------------------------------------ exact fp32
def round_f32(v: Fraction) -> Fraction:
    """Nearest binary32 to the exact rational v (ties to even); no overflow handling."""
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    # exponent e with 2^e <= a < 2^(e+1)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -126)               # below 2^-126 the spacing is fixed (subnormals)
    ulp = Fraction(2) ** (e - 23)
    m = a / ulp
    lo = m.numerator // m.denominator
    rem = m - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return sign * lo * ulp


def f32(x: float) -> Fraction:
    """Exact value of a Python float that is already a binary32 value."""
    return Fraction(x)


def bf16_bits_to_fraction(bits: int) -> Fraction:
    return Fraction(struct.unpack("<f", struct.pack("<I", (bits & 0xFFFF) << 16))[0])


def fp16_bits_to_float(bits: int) -> float:
    return float(struct.unpack("<e", struct.pack("<H", bits & 0xFFFF))[0])


# ------------------------------------------------------------ router
def router_logit(x_bits, w, bias=None) -> Fraction:
    """Fixed-order fp32 logit: 32 fma chains over chunks of 128, pairwise tree, bias."""
    d = len(x_bits)
    acc = [Fraction(0)] * 32
    for i in range(d // 128):
        for lane in range(32):
            for j in range(4):
                kk = 128 * i + 4 * lane + j
                acc[lane] = round_f32(bf16_bits_to_fraction(x_bits[kk]) * f32(w[kk]) + acc[lane])
    o = 16
    while o >= 1:
        acc = [round_f32(acc[lane] + acc[lane ^ o]) for lane in range(32)]
        o //= 2
    r = acc[0]
    if bias is not None:
        r = round_f32(r + f32(bias))
    return r


def topk(logits_row, k):
    """Best k-subset by exact logit sum; ties to the smallest sorted id tuple."""
    best, best_sum = None, None
    for sub in itertools.combinations(range(len(logits_row)), k):
        s = sum(Fraction(logits_row[e]) for e in sub)
        if best_sum is None or s > best_sum:
            best, best_sum = sub, s
    mx = max(float(logits_row[e]) for e in best)
    ex = [math.exp(float(logits_row[e]) - mx) for e in best]
    z = sum(ex)
    return list(best), [v / z for v in ex]


def permute(idx_rows, E):
    k = len(idx_rows[0]) if idx_rows else 0
    pairs = [(idx_rows[p // k][p % k], p) for p in range(len(idx_rows) * k)]
    order = sorted(pairs)
    counts = [0] * E
    for e, _ in order:
        counts[e] += 1
    offsets = [0]
    for e in range(E):
        offsets.append(offsets[-1] + counts[e])
    inv = [0] * len(order)
    for s, (_, p) in enumerate(order):
        inv[p] = s
    return {"counts": counts, "offsets": offsets, "sorted_tok": [p // k for _, p in order],
            "sorted_j": [p % k for _, p in order], "inv": inv,
            "active": [e for e in range(E) if counts[e] > 0]}


def cache_lookup(slot_of, layer, idx_rows, gate_rows):
    sop = [slot_of[e] for row in idx_rows for e in row]
    misses = []
    for e in sorted(set(e for row in idx_rows for e in row)):
        if slot_of[e] >= 0:
            continue
        for t, row in enumerate(idx_rows):
            for j, ee in enumerate(row):
                if ee == e:
                    misses.append((layer, e, t, j, gate_rows[t][j]))
    return sop, misses


# ------------------------------------------------------------ dequant + FFN
def _bit(buf_row, bitpos):
    return (int(buf_row[bitpos // 8]) >> (bitpos % 8)) & 1


def dequant(mat, fmt):
    codes = mat["codes"]
    R, K = len(codes), len(codes[0]) * 4
    W = [[0.0] * K for _ in range(R)]
    for r in range(R):
        for k in range(K):
            q = _bit(codes[r], 2 * k) + 2 * _bit(codes[r], 2 * k + 1)
            s = fp16_bits_to_float(int(mat["scale"][r][k // 64]))
            if fmt == 2:
                W[r][k] = s * q + fp16_bits_to_float(int(mat["min"][r][k // 64]))
            else:
                q += 4 * _bit(mat["hi"][r], k)
                W[r][k] = s * (q - 4)
    return W


def ffn(W, x):
    f, d = len(W["gate"]), len(x)
    h = []
    for r in range(f):
        a = sum(W["gate"][r][c] * x[c] for c in range(d))
        u = sum(W["up"][r][c] * x[c] for c in range(d))
        h.append(a / (1.0 + math.exp(-a)) * u)
    return [sum(W["down"][r][c] * h[c] for c in range(f)) for r in range(d)]


def layer(x_bits, Wr, bias, experts, shared, k, fmt, slot_of=None, fmt_of=None):
    T, d = len(x_bits), len(x_bits[0])
    E = len(Wr)
    logits = [[router_logit(x_bits[t], Wr[e], None if bias is None else bias[e]) for e in range(E)]
              for t in range(T)]
    sel = [topk([float(v) for v in logits[t]], k) for t in range(T)]
    idx = [s[0] for s in sel]
    gate = [s[1] for s in sel]
    if slot_of is None:
        slot_of = list(range(E))
    xf = [[float(bf16_bits_to_fraction(b)) for b in row] for row in x_bits]
    Wsh = {m: dequant(shared[m], fmt) for m in ("gate", "up", "down")}
    Wd = {}
    y_part, y_full = [], []
    for t in range(T):
        acc = ffn(Wsh, xf[t])
        full = list(acc)
        for j in range(k):
            e = idx[t][j]
            if e not in Wd:
                fe = fmt if fmt_of is None else fmt_of[e]
                Wd[e] = {m: dequant(experts[e][m], fe) for m in ("gate", "up", "down")}
            ye = ffn(Wd[e], xf[t])
            full = [a + gate[t][j] * b for a, b in zip(full, ye)]
            if slot_of[e] >= 0:
                acc = [a + gate[t][j] * b for a, b in zip(acc, ye)]
        y_part.append(acc)
        y_full.append(full)
    return {"logits": logits, "idx": idx, "gate": gate, "perm": permute(idx, E),
            "y_partial": y_part, "y_full": y_full}
