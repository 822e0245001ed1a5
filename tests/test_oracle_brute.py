"""The C oracle against the pure-Python brute force on tiny layers (CPU only).

The brute force does fp32 arithmetic exactly with fractions and one rounding,
enumerates every k-subset for top-k, sorts pairs with sorted() and runs the FFN
in Python loops -- an independent statement of the same layer.
"""
import numpy as np
import pytest

from bit_expert_ffn_fp32_b200 import synth


def _tiny(fmt, seed, T=3, d=128, E=8, f=64, bias=True, ties=False):
    x = synth.gen_x(seed, 0, T, d)
    Wr = synth.gen_router(seed, 0, E, d)
    if ties:
        Wr[3] = Wr[1]           # experts 1 and 3 always tie
        Wr[6] = Wr[1]
    b = synth.zipf_bias(synth.gen_rank_perm(seed, 0, E), 0.5) if bias else None
    if ties and b is not None:
        b[3] = b[1]
        b[6] = b[1]
    experts = {e: synth.gen_expert(seed, 0, e, fmt, d, f) for e in range(E)}
    shared = synth.gen_expert(seed, 0, E, fmt, d, f)
    return x, Wr, b, experts, shared


@pytest.mark.parametrize("fmt,seed,bias,ties", [(2, 0, True, False), (3, 1, True, False), (2, 2, False, True),
                                                (3, 3, True, True)])
def test_layer_vs_brute(orc, brute, fmt, seed, bias, ties):
    k, E = 3, 8
    x, Wr, b, experts, shared = _tiny(fmt, seed, bias=bias, ties=ties)
    slot_of = np.array([0, 1, -1, 2, 3, -1, 4, 5], np.int32)
    o = orc.layer(x, Wr, b, experts.__getitem__, shared, k, fmt, slot_of=slot_of, layer_id=1)
    br = brute.layer(x.tolist(), Wr.tolist(), None if b is None else b.tolist(),
                     {e: {m: {kk: (None if v is None else v.tolist()) for kk, v in experts[e][m].items()}
                          for m in experts[e]} for e in experts},
                     {m: {kk: (None if v is None else v.tolist()) for kk, v in shared[m].items()} for m in shared},
                     k, fmt, slot_of=slot_of.tolist())
    # fp32 logits bit-exact
    np.testing.assert_array_equal(o["logit32"], np.array([[float(v) for v in row] for row in br["logits"]],
                                                         np.float32))
    np.testing.assert_array_equal(o["idx"], np.array(br["idx"]))
    np.testing.assert_allclose(o["gate"], np.array(br["gate"]), rtol=1e-13)
    for key in ("counts", "offsets", "sorted_tok", "sorted_j", "inv"):
        np.testing.assert_array_equal(o["perm"][key], np.array(br["perm"][key]), err_msg=key)
    act = br["perm"]["active"]
    assert o["perm"]["active"][0] == len(act)
    np.testing.assert_array_equal(o["perm"]["active"][1:1 + len(act)], act)
    sop, misses = brute.cache_lookup(slot_of.tolist(), 1, br["idx"], br["gate"])
    np.testing.assert_array_equal(o["slot_of_pair"], sop)
    assert [m[:4] for m in o["misses"]] == [m[:4] for m in misses]
    np.testing.assert_allclose(o["y_partial"], np.array(br["y_partial"]), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(o["y_full"], np.array(br["y_full"]), rtol=1e-10, atol=1e-12)


def test_mixed_format_layer_vs_brute(orc, brute):
    """A pool holding both tiers: each routed expert dequantised by its own
    format (Q3 for the odd ids, Q2 for the rest, shared Q2), the oracle against
    the brute force; and the routed part differs from the all-Q2 layer exactly
    where a Q3 expert was routed."""
    k, E, d, f, seed = 3, 8, 128, 64, 5
    x, Wr, b, _, shared = _tiny(2, seed)
    fmt_of = [3 if e % 2 else 2 for e in range(E)]
    experts = {e: synth.gen_expert(seed, 0, e, fmt_of[e], d, f) for e in range(E)}
    slot_of = np.array([0, 1, 2, -1, 3, 4, -1, 5], np.int32)
    o = orc.layer(x, Wr, b, experts.__getitem__, shared, k, 2, slot_of=slot_of, fmt_of=np.array(fmt_of))
    lst = lambda m: {kk: (None if v is None else v.tolist()) for kk, v in m.items()}
    br = brute.layer(x.tolist(), Wr.tolist(), b.tolist(),
                     {e: {m: lst(experts[e][m]) for m in experts[e]} for e in experts},
                     {m: lst(shared[m]) for m in shared}, k, 2, slot_of=slot_of.tolist(), fmt_of=fmt_of)
    np.testing.assert_array_equal(o["idx"], np.array(br["idx"]))
    np.testing.assert_allclose(o["y_partial"], np.array(br["y_partial"]), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(o["y_full"], np.array(br["y_full"]), rtol=1e-10, atol=1e-12)
    assert any(fmt_of[int(e)] == 3 for e in o["idx"].ravel())
    q2 = {e: synth.gen_expert(seed, 0, e, 2, d, f) for e in range(E)}
    o2 = orc.layer(x, Wr, b, q2.__getitem__, shared, k, 2, slot_of=slot_of)
    for t in range(x.shape[0]):
        same = all(fmt_of[int(e)] == 2 for e in o["idx"][t])
        assert np.array_equal(o["y_full"][t], o2["y_full"][t]) == same


def test_round_f32_matches_numpy(brute):
    from fractions import Fraction
    rng = np.random.default_rng(0)
    vals = np.concatenate([rng.standard_normal(300) * 10.0 ** rng.integers(-40, 30, 300), [1e-45, 3e-39, 2.0 ** 24 + 1]])
    for v in vals:
        assert float(brute.round_f32(Fraction(float(v)))) == float(np.float32(v)), v


def test_dequant_brute_vs_oracle(orc, brute):
    for fmt in (2, 3):
        m = synth.gen_matrix(9, 0, 0, "gate", fmt, 5, 192)
        W = orc.dequant(m, fmt)
        Wb = brute.dequant({kk: (None if v is None else v.tolist()) for kk, v in m.items()}, fmt)
        np.testing.assert_array_equal(W, np.array(Wb))
