"""Pins of the CPU oracle against facts fixed outside it (CPU only).

Each test checks one oracle function against something other than itself:
number-format definitions, hand-made quantised rows, hand-derived fp32
operation-order cases, closed forms, library routines (torch float64), brute
force, invariants, or figures the pages print.
"""
import math

import numpy as np
import pytest
import torch

from conftest import golden_rows
from bit_expert_ffn_fp32_b200 import configs, synth


# ------------------------------------------------------------------ formats
def test_number_formats(orc):
    for kind, hexbits, val in golden_rows("number_formats.txt"):
        got = orc.bf16_value(int(hexbits, 16)) if kind == "bf16" else orc.fp16_value(int(hexbits, 16))
        assert got == float(val), (kind, hexbits, got, val)
        assert math.copysign(1.0, got) == math.copysign(1.0, float(val))


def _parse_bytes(spec, n):
    buf = np.zeros(n, np.uint8)
    if spec != "-":
        for item in spec.split(","):
            i, v = item.split(":")
            buf[int(i)] = int(v, 16)
    return buf


@pytest.mark.parametrize("row", golden_rows("quant_blocks.txt"), ids=lambda r: f"{r[0]}_{r[1]}")
def test_dequant_golden(orc, row):
    fmt_s, K, codes_s, hi_s, sc_s, mn_s, w_s, dflt_s = row
    fmt, K = (2 if fmt_s == "q2" else 3), int(K)
    codes = _parse_bytes(codes_s, K // 4)[None, :]
    hi = _parse_bytes(hi_s, K // 8)[None, :] if fmt == 3 else None
    scale = np.array([[int(h, 16) for h in sc_s.split(",")]], np.uint16)
    mn = np.array([[int(h, 16) for h in mn_s.split(",")]], np.uint16) if fmt == 2 else None
    W = orc.dequant(synth.matrix_from_parts(codes, scale, mn, hi), fmt)[0]
    dflt = [float(v) for v in dflt_s.split(",")]
    expect = np.array([dflt[k // 64] for k in range(K)])
    for item in w_s.split(","):
        i, v = item.split(":")
        expect[int(i)] = float(v)
    np.testing.assert_array_equal(W, expect)


def test_dequant_zero_scale_is_block_min(orc):
    rng = np.random.default_rng(3)
    R, K = 4, 256
    codes = rng.integers(0, 256, (R, K // 4), dtype=np.uint8)
    scale = np.zeros((R, K // 64), np.uint16)
    mn = synth.f32_to_fp16_bits(rng.normal(0, 0.01, (R, K // 64)))
    W = orc.dequant(synth.matrix_from_parts(codes, scale, mn), 2)
    mvals = mn.view(np.float16).astype(np.float64)
    np.testing.assert_array_equal(W, np.repeat(mvals, 64, axis=1))
    # closed form W x = sum_b m_b * sum_{k in b} x_k (fp64 library matmul for the sum)
    x = rng.standard_normal(K)
    np.testing.assert_allclose(W @ x, (mvals * x.reshape(K // 64, 64).sum(1)[None, :]).sum(1), rtol=1e-12)


def test_q3_code4_is_zero(orc):
    R, K = 3, 128
    lo = np.zeros((R, K // 4), np.uint8)
    hi = np.full((R, K // 8), 0xFF, np.uint8)
    scale = synth.f32_to_fp16_bits(np.full((R, K // 64), 0.37))
    W = orc.dequant(synth.matrix_from_parts(lo, scale, None, hi), 3)
    assert np.all(W == 0.0)


# ------------------------------------------------------------------ router
@pytest.mark.parametrize("row", golden_rows("router_order_cases.txt"), ids=lambda r: r[0])
def test_router_operation_order(orc, row):
    name, d, elems, bias, expect, _why = row
    d = int(d)
    x = np.zeros(d, np.uint16)
    w = np.zeros(d, np.float32)
    for item in elems.split(","):
        i, v = item.split(":")
        x[int(i)] = 0x3F80
        w[int(i)] = float(v)
    b = None if bias == "-" else float(bias)
    got = orc.router_logit(x, w, b)
    assert got == np.float32(float(expect)), (name, got)


def test_router_small_integers_exact(orc):
    # x and w small integers: every product and partial sum is an exact fp32
    # integer, so the fixed-order fp32 logit equals the exact integer dot product.
    rng = np.random.default_rng(5)
    T, d, E = 3, 512, 7
    xi = rng.integers(-8, 9, (T, d))
    wi = rng.integers(-8, 9, (E, d))
    x = synth.f32_to_bf16_bits(xi.astype(np.float32))
    l32, _, _ = orc.router(x, wi.astype(np.float32), None)
    np.testing.assert_array_equal(l32.astype(np.int64), xi @ wi.T)


@pytest.mark.parametrize("wl", [configs.TINY, configs.DECODE])
def test_router_within_rounding_bound(orc, wl):
    x = synth.gen_x(11, 0, 8, wl.d)
    Wr = synth.gen_router(11, 0, wl.E, wl.d)
    bias = synth.zipf_bias(synth.gen_rank_perm(11, 0, wl.E), configs.ZIPF_ALPHA) if wl.zipf else None
    l32, l64, ad = orc.router(x, Wr, bias)
    # l64 against a library fp64 product
    xf = orc.bf16_to_f64(x)
    ref = xf @ Wr.astype(np.float64).T + (0 if bias is None else bias.astype(np.float64)[None, :])
    np.testing.assert_allclose(l64, ref, rtol=0, atol=1e-11)
    bound = orc.logit_error_bound(wl.d, ad, bias)
    assert np.all(np.abs(l32.astype(np.float64) - ref) <= bound)


# ------------------------------------------------------------------ top-k and gates
def test_topk_ties_lowest_index(orc):
    logits = np.zeros((2, 9), np.float32)
    logits[1, :] = -0.0            # -0 and +0 compare equal
    logits[1, 4] = 0.0
    idx, g = orc.topk(logits, 4)
    np.testing.assert_array_equal(idx, [[0, 1, 2, 3], [0, 1, 2, 3]])
    np.testing.assert_allclose(g, 0.25, rtol=0, atol=1e-15)


def test_topk_order_and_ascending_output(orc):
    logits = np.array([[0.5, 3.0, -1.0, 3.0, 2.0, 0.5]], np.float32)
    idx, g = orc.topk(logits, 4)
    np.testing.assert_array_equal(idx, [[0, 1, 3, 4]])   # 3.0, 3.0, 2.0, then 0.5 at id 0 (not 5)
    z = 2 * math.exp(0) + math.exp(-1.0) + math.exp(-2.5)
    np.testing.assert_allclose(g[0], [math.exp(-2.5) / z, 1 / z, 1 / z, math.exp(-1.0) / z], rtol=1e-14)


def test_gates_closed_form_two_experts(orc):
    l = np.array([[0.0, np.float32(math.log(3.0)), -5.0, -6.0]], np.float32)
    _, g = orc.topk(l, 2)
    np.testing.assert_allclose(g[0], [0.25, 0.75], rtol=1e-7)


def test_gates_one_hot(orc):
    l = np.zeros((1, 16), np.float32)
    l[0, 9] = 800.0
    idx, g = orc.topk(l, 3)
    np.testing.assert_array_equal(idx[0], [0, 1, 9])
    np.testing.assert_array_equal(g[0], [0.0, 0.0, 1.0])


def test_topk_matches_full_softmax_renormalised(orc):
    rng = np.random.default_rng(8)
    l = rng.standard_normal((5, 64)).astype(np.float32)
    idx, g = orc.topk(l, 6)
    full = torch.softmax(torch.from_numpy(l.astype(np.float64)), dim=1).numpy()
    sel = np.take_along_axis(full, idx.astype(np.int64), axis=1)
    np.testing.assert_allclose(g, sel / sel.sum(1, keepdims=True), rtol=1e-13)
    np.testing.assert_allclose(g.sum(1), 1.0, rtol=0, atol=1e-12)
    # the selection is the k largest (library sort, ties impossible here)
    ref = np.sort(np.argsort(-l, axis=1, kind="stable")[:, :6], axis=1)
    np.testing.assert_array_equal(idx, ref)


def test_topk_rejects_nonfinite(orc):
    l = np.zeros((1, 8), np.float32)
    l[0, 3] = np.nan
    with pytest.raises(ValueError):
        orc.topk(l, 2)


# ------------------------------------------------------------------ permutation / cache
def test_permute_invariants_and_library_sort(orc):
    rng = np.random.default_rng(2)
    T, E, k = 50, 40, 6
    idx = np.sort(np.stack([rng.choice(E, k, replace=False) for _ in range(T)]), axis=1).astype(np.int32)
    p = orc.permute(idx, E)
    n = T * k
    assert p["counts"].sum() == n and p["offsets"][-1] == n
    np.testing.assert_array_equal(np.sort(p["inv"]), np.arange(n))        # bijection
    flat = idx.ravel()
    order = np.lexsort((np.arange(n), flat))                                 # library stable sort
    np.testing.assert_array_equal(p["sorted_tok"] * k + p["sorted_j"], order)
    np.testing.assert_array_equal(p["inv"][order], np.arange(n))
    np.testing.assert_array_equal(p["counts"], np.bincount(flat, minlength=E))
    act = np.flatnonzero(p["counts"])
    assert p["active"][0] == len(act)
    np.testing.assert_array_equal(p["active"][1:1 + len(act)], act)


def test_cache_lookup_invariants(orc):
    rng = np.random.default_rng(4)
    T, E, k = 30, 32, 4
    idx = np.sort(np.stack([rng.choice(E, k, replace=False) for _ in range(T)]), axis=1).astype(np.int32)
    gate = rng.random((T, k))
    slot_of = np.where(rng.random(E) < 0.5, np.arange(E) + 100, -1).astype(np.int32)
    sop, miss, n = orc.cache_lookup(slot_of, 7, idx, gate, E)
    np.testing.assert_array_equal(sop, slot_of[idx.ravel()])
    assert n == int((sop < 0).sum()) and len(miss) == n
    keys = [(m[1], m[2]) for m in miss]
    assert keys == sorted(keys)
    for (lay, e, t, j, g) in miss:
        assert lay == 7 and idx[t, j] == e and slot_of[e] < 0 and g == np.float32(gate[t, j])
    _, miss2, n2 = orc.cache_lookup(slot_of, 7, idx, gate, E, miss_cap=3)
    assert n2 == n and miss2 == miss[:3]


# ------------------------------------------------------------------ experts
def _identity_expert(d):
    """Q2 expert with Wg = I, Wu = 2I, Wd = I on a d x d block."""
    def mat(q):
        codes = np.zeros((d, d // 4), np.uint8)
        for r in range(d):
            codes[r, r // 4] |= q << (2 * (r % 4))
        scale = np.full((d, d // 64), 0x3C00, np.uint16)
        mn = np.zeros((d, d // 64), np.uint16)
        return synth.matrix_from_parts(codes, scale, mn)
    return {"gate": mat(1), "up": mat(2), "down": mat(1)}


def test_swiglu_closed_form(orc):
    rows = golden_rows("swiglu_identity.txt")
    d = 64
    W = orc.dequant_expert(_identity_expert(d), 2)
    x = np.zeros(d)
    for i, (xv, _) in enumerate(rows):
        x[i] = float(xv)
    y = orc.expert_ffn(W, x)[0]
    for i, (_, yv) in enumerate(rows):
        assert y[i] == pytest.approx(float(yv), rel=1e-14, abs=1e-300)


def test_expert_ffn_matches_torch(orc):
    rng_seed = 21
    d, f = 256, 128
    ex = synth.gen_expert(rng_seed, 0, 0, 2, d, f)
    W = orc.dequant_expert(ex, 2)
    x = orc.bf16_to_f64(synth.gen_x(rng_seed, 0, 3, d))
    y = orc.expert_ffn(W, x)
    tW = {m: torch.from_numpy(W[m]) for m in W}
    tx = torch.from_numpy(x)
    a = tx @ tW["gate"].T
    u = tx @ tW["up"].T
    ref = (torch.nn.functional.silu(a) * u) @ tW["down"].T
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ whole layer
def _small_layer(fmt, seed=0, T=4, d=256, E=8, f=128, k=3, zero_routed=False):
    experts = {e: synth.gen_expert(seed, 0, e, fmt, d, f) for e in range(E)}
    if zero_routed:
        for e in experts:
            for m in experts[e].values():
                m["codes"][:] = 0
                if fmt == 2:
                    m["min"][:] = 0
                else:
                    m["hi"][:] = 0xFF        # q = 4 everywhere -> w = 0
    shared = synth.gen_expert(seed, 0, E, fmt, d, f)
    x = synth.gen_x(seed, 0, T, d)
    Wr = synth.gen_router(seed, 0, E, d)
    return x, Wr, experts, shared


@pytest.mark.parametrize("fmt", [2, 3])
def test_layer_zero_routed_gives_shared(orc, fmt):
    x, Wr, experts, shared = _small_layer(fmt, zero_routed=True)
    out = orc.layer(x, Wr, None, experts.__getitem__, shared, 3, fmt)
    ysh = orc.expert_ffn(orc.dequant_expert(shared, fmt), orc.bf16_to_f64(x))
    np.testing.assert_array_equal(out["y_partial"], ysh)


def test_layer_zero_input(orc):
    x, Wr, experts, shared = _small_layer(2)
    x[:] = 0
    out = orc.layer(x, Wr, None, experts.__getitem__, shared, 3, 2)
    np.testing.assert_array_equal(out["idx"], np.tile([0, 1, 2], (x.shape[0], 1)))
    np.testing.assert_allclose(out["gate"], 1 / 3, rtol=1e-15)
    assert np.all(out["y_partial"] == 0)


def test_layer_one_hot_router_is_dense_expert(orc):
    # one expert's bias dominates: its gate is exactly 1 and the others exactly 0
    x, Wr, experts, shared = _small_layer(2, T=3)
    bias = np.zeros(Wr.shape[0], np.float32)
    bias[5] = 800.0
    out = orc.layer(x, Wr, bias, experts.__getitem__, shared, 3, 2)
    xt = torch.from_numpy(orc.bf16_to_f64(x))

    def dense(ex):
        W = {m: torch.from_numpy(orc.dequant(ex[m], 2)) for m in ex}
        return ((torch.nn.functional.silu(xt @ W["gate"].T) * (xt @ W["up"].T)) @ W["down"].T).numpy()

    for t in range(x.shape[0]):
        row = list(out["idx"][t])
        assert 5 in row
        np.testing.assert_array_equal(out["gate"][t], [1.0 if e == 5 else 0.0 for e in row])
    np.testing.assert_allclose(out["y_partial"], dense(shared) + dense(experts[5]), rtol=1e-11, atol=1e-12)


def test_layer_full_equals_partial_plus_misses(orc):
    x, Wr, experts, shared = _small_layer(3, T=6)
    slot_of = np.array([0, -1, 1, -1, 2, 3, -1, 4], np.int32)
    out = orc.layer(x, Wr, None, experts.__getitem__, shared, 3, 3, slot_of=slot_of, layer_id=2)
    xf = orc.bf16_to_f64(x)
    add = np.zeros_like(out["y_full"])
    for (_, e, t, j, _g) in out["misses"]:
        add[t] += out["gate"][t, j] * orc.expert_ffn(orc.dequant_expert(experts[e], 3), xf[t])[0]
    np.testing.assert_allclose(out["y_full"], out["y_partial"] + add, rtol=1e-12, atol=1e-13)
    assert out["miss_count"] == int(np.isin(out["idx"], [1, 3, 6]).sum())


# ------------------------------------------------------------------ facts the pages print
def test_page_facts():
    facts = {r[0]: float(r[1]) for r in golden_rows("page_facts.txt")}
    wl = configs.DECODE
    assert wl.E == facts["experts_per_layer"] and wl.k == facts["routed_per_token"]
    assert configs.STACK48.layers * wl.E == facts["experts_total"]
    assert abs(100 * wl.k / wl.E - facts["active_fraction_pct"]) < 0.1
    per_gb = 1e9 / configs.expert_bytes(2, wl.d, wl.f)
    assert abs(per_gb / facts["experts_per_GB"] - 1) < 0.10
    res = configs.STACK48.resident * configs.STACK48.layers
    assert res / facts["experts_total"] == facts["resident_fraction"]
    assert abs(res / facts["resident_experts_max"] - 1) < 0.05
    assert configs.VERIFY.T == 1 + facts["mtp_draft_tokens"]
    assert configs.PREFILL.T == facts["prefill_chunk_max"]
    # the page's IQ3_XXS cache: bytes per weight sit between our Q2 and Q3 formats
    bpw = facts["cache_GB"] * 8e9 / facts["cache_experts"] / (3 * wl.d * wl.f)
    assert 2.5 < bpw < 3.25
