"""Randomised (hypothesis) parity of the host components against their oracles:
the cache policy's plans equal the oracle's for random shapes, parameters and
traces; the host miss completion matches the fp64 oracle for random shapes,
formats and record lists. Derandomised, so every run draws the same cases."""
import numpy as np
from hypothesis import given, settings, strategies as st

from bit_expert_ffn_fp32_b200 import native, synth
from policy import PolicyOracle

MISS_DT = np.dtype([("layer", "<i4"), ("expert", "<i4"), ("token", "<i4"), ("j", "<i4"), ("gate", "<f4")])


@settings(max_examples=40, deadline=None, derandomize=True)
@given(L=st.integers(1, 3), E=st.integers(2, 24), slots_frac=st.floats(0.0, 1.0), k=st.integers(1, 4),
       epoch=st.integers(1, 40), margin=st.integers(0, 3), max_swaps=st.integers(0, 10),
       plan_every=st.integers(1, 6), seed=st.integers(0, 1000))
def test_policy_equals_oracle_random(L, E, slots_frac, k, epoch, margin, max_swaps, plan_every, seed):
    k = min(k, E)
    S = int(slots_frac * L * E)
    trace = synth.gen_routing_trace(seed, L, E, k, 40, drift_every=7, drift_swaps=2)
    lib = native.CachePolicy(L, E, S, epoch, margin)
    orc = PolicyOracle(L, E, S, epoch, margin)
    slot_lib = np.full((L, E), -1, np.int32)
    slot_orc = [[-1] * E for _ in range(L)]
    rng = np.random.default_rng(seed)
    for t in range(trace.shape[0]):
        for l in range(L):
            n_tok = int(rng.integers(1, 3))  # one or two tokens per call
            rows = np.repeat(trace[t, l][None, :], n_tok, axis=0)
            lib.observe(l, rows)
            orc.observe(l, rows.tolist())
        if (t + 1) % plan_every == 0:
            assert lib.plan(slot_lib, max_swaps) == orc.plan(slot_orc, max_swaps)
            np.testing.assert_array_equal(slot_lib, np.array(slot_orc, np.int32))


@settings(max_examples=12, deadline=None, derandomize=True)
@given(fmt=st.sampled_from([2, 3]), d=st.sampled_from([256, 512]), f=st.sampled_from([256, 512]),
       T=st.integers(1, 4), n=st.integers(1, 6), nthreads=st.integers(0, 3), seed=st.integers(0, 1000))
def test_miss_completion_matches_oracle_random(orc, fmt, d, f, T, n, nthreads, seed):
    rng = np.random.default_rng(seed)
    E = 5
    canon = {e: synth.gen_expert(seed, 0, e, fmt, d, f) for e in range(E)}
    tab = native.expert_table(E, canon)
    x = synth.gen_x(seed, 0, T, d, stream=3)
    recs = np.array([(0, int(rng.integers(0, E)), int(rng.integers(0, T)), int(rng.integers(0, 10)),
                      float(rng.uniform(0.0, 1.0))) for _ in range(n)], MISS_DT)
    y = np.zeros((T, d), np.float32)
    native.complete_misses_host(fmt, d, f, tab, E, recs, n, 0, x, T, y, nthreads)
    xf = orc.bf16_to_f64(x)
    ref = np.zeros((T, d))
    for r in recs:
        W = orc.dequant_expert(canon[int(r["expert"])], fmt)
        ref[int(r["token"])] += float(r["gate"]) * orc.expert_ffn(W, xf[int(r["token"])])[0]
    scale = max(np.max(np.abs(ref)), 1e-30)
    assert np.max(np.abs(y - ref)) / scale <= 1e-5
