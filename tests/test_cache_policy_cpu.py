"""Expert-cache policy (moe_cache_policy_*) against its oracle and against
facts that do not depend on either: the resident set after a full plan on a
stationary count table is the top-S set computed by a sort of numpy counts,
counts halve per epoch, no improving swap is left, and slot tables stay
partial injections. Under drifting popularity the online policy keeps a higher
hit rate than a resident set fixed from early counts (the pages' point: 72%
against 50% for a frequency curve)."""
import numpy as np
import pytest

from bit_expert_ffn_fp32_b200 import native, synth
from policy import PolicyOracle


def _check_injection(slot_of, S):
    held = slot_of[slot_of >= 0]
    assert len(set(held.tolist())) == len(held) and np.all(held < S)


def _replay(L, E, S, epoch, margin, trace, plan_every, max_swaps):
    """Run the library and the oracle side by side; returns the library's slot
    table history and checks every plan for equality."""
    lib = native.CachePolicy(L, E, S, epoch, margin)
    orc = PolicyOracle(L, E, S, epoch, margin)
    slot_lib = np.full((L, E), -1, np.int32)
    slot_orc = [[-1] * E for _ in range(L)]
    hits = total = 0
    for t in range(trace.shape[0]):
        for l in range(L):
            rows = trace[t, l][None, :]
            hits += int((slot_lib[l][rows[0]] >= 0).sum())
            total += rows.shape[1]
            lib.observe(l, rows)
            orc.observe(l, rows.tolist())
        if (t + 1) % plan_every == 0:
            sw_lib = lib.plan(slot_lib, max_swaps)
            sw_orc = orc.plan(slot_orc, max_swaps)
            assert sw_lib == sw_orc
            np.testing.assert_array_equal(slot_lib, np.array(slot_orc, np.int32))
            _check_injection(slot_lib, S)
    return hits / total


@pytest.mark.parametrize("epoch,margin,max_swaps", [(64, 0, 4), (16, 2, 1), (1000, 1, 64)])
def test_policy_matches_oracle_on_drifting_trace(epoch, margin, max_swaps):
    L, E, S, k = 3, 32, 24, 4
    trace = synth.gen_routing_trace(4, L, E, k, 300, drift_every=40, drift_swaps=6)
    _replay(L, E, S, epoch, margin, trace, plan_every=5, max_swaps=max_swaps)


def test_full_plan_on_stationary_counts_keeps_the_top_s():
    """No halving within the run, margin 0, unlimited swaps: the resident set is
    the S (layer, expert) with the largest counts (ties to the lower index),
    computed here with numpy from the trace."""
    L, E, S, k = 2, 40, 17, 3
    trace = synth.gen_routing_trace(8, L, E, k, 150)
    pol = native.CachePolicy(L, E, S, epoch=10**6, margin=0)
    for t in range(trace.shape[0]):
        for l in range(L):
            pol.observe(l, trace[t, l][None, :])
    slot = np.full((L, E), -1, np.int32)
    slot[0, :5] = np.arange(5)  # a stale start: arbitrary experts in slots 0..4
    pol.plan(slot, 10**6)
    pol.plan(slot, 10**6)       # a second plan changes nothing
    cnt = np.zeros(L * E, np.int64)
    for l in range(L):
        cnt[l * E:(l + 1) * E] = np.bincount(trace[:, l].ravel(), minlength=E)
    order = sorted(range(L * E), key=lambda i: (-cnt[i], i))
    top = set(i for i in order[:S] if cnt[i] > 0)
    resident = set(np.flatnonzero(slot.ravel() >= 0).tolist())
    # equal counts at the boundary may resolve either way only through the index rule
    assert resident == top
    _check_injection(slot, S)


def test_halving_per_epoch_and_margin():
    L, E, S = 1, 8, 1
    pol = native.CachePolicy(L, E, S, epoch=4, margin=3)
    slot = np.full((L, E), -1, np.int32)
    pol.observe(0, np.array([[1, 2]] * 3, np.int32))    # counts e1 = e2 = 3, clock 3
    assert pol.plan(slot, 8) == [(0, 0, 1, -1, -1)]     # free slot to the lower id
    pol.observe(0, np.array([[2, 3]] * 3, np.int32))    # clock 6: halve (1, 1) then e2 = 4, e3 = 3
    assert pol.plan(slot, 8) == []                      # 4 > 1 + 3 is false: margin holds e1
    pol.observe(0, np.array([[2, 3]], np.int32))        # clock 7: e2 = 5 > 1 + 3
    assert pol.plan(slot, 8) == [(0, 0, 2, 0, 1)]
    _check_injection(slot, S)


def test_no_improving_swap_left_after_a_full_plan():
    L, E, S, k = 2, 30, 12, 3
    margin = 2
    trace = synth.gen_routing_trace(2, L, E, k, 120, drift_every=30, drift_swaps=5)
    pol = native.CachePolicy(L, E, S, epoch=50, margin=margin)
    orc = PolicyOracle(L, E, S, epoch=50, margin=margin)
    slot = np.full((L, E), -1, np.int32)
    for t in range(trace.shape[0]):
        for l in range(L):
            pol.observe(l, trace[t, l][None, :])
            orc.observe(l, [trace[t, l].tolist()])
    pol.plan(slot, 10**6)
    cnt = np.array(orc.count).ravel()
    res = slot.ravel() >= 0
    if res.any() and (~res).any():
        assert cnt[~res].max() <= cnt[res].min() + margin
    assert res.sum() == min(S, int((cnt > 0).sum()))  # free slots all went to used experts


def test_invalid_slot_table_and_state_are_rejected():
    pol = native.CachePolicy(1, 4, 2, epoch=8)
    bad = np.array([[0, 0, -1, -1]], np.int32)          # slot 0 twice
    with pytest.raises(native.MoeError):
        pol.plan(bad, 4)
    np.testing.assert_array_equal(bad, [[0, 0, -1, -1]])
    with pytest.raises(native.MoeError):
        pol.plan(np.array([[2, -1, -1, -1]], np.int32), 4)  # slot outside [0, S)
    with pytest.raises(native.MoeError):
        pol.observe(0, np.array([[4]], np.int32))       # expert outside [0, E)
    assert native.lib.moe_cache_policy_bytes(0, 4) == 0


def test_online_policy_beats_a_fixed_frequency_set_under_drift():
    """Drifting Zipf(1.1) popularity, a quarter of the experts resident: the
    online policy's hit rate exceeds that of the set chosen from the first
    window's counts and never changed."""
    L, E, k, n = 4, 64, 4, 1200
    S = L * E // 4
    trace = synth.gen_routing_trace(6, L, E, k, n, drift_every=100, drift_swaps=16)
    online = _replay(L, E, S, epoch=64, margin=1, trace=trace, plan_every=8, max_swaps=8)
    warm = 100
    cnt = np.stack([np.bincount(trace[:warm, l].ravel(), minlength=E) for l in range(L)]).ravel()
    fixed = np.zeros(L * E, bool)
    fixed[sorted(range(L * E), key=lambda i: (-cnt[i], i))[:S]] = True
    fixed = fixed.reshape(L, E)
    hits = sum(int(fixed[l][trace[t, l]].sum()) for t in range(n) for l in range(L))
    fixed_rate = hits / (n * L * k)
    assert online > fixed_rate + 0.05, (online, fixed_rate)


def test_cache_sim_tool_small():
    from bit_expert_ffn_fp32_b200 import cache_sim

    r = cache_sim.simulate(L=2, E=16, S=8, k=2, tokens=60, s=1.1, drift_every=20, drift_swaps=3, epoch=16,
                           margin=0, plan_every=4, max_swaps=4, warm=10)
    assert 0.0 <= r["fixed_hit_rate"] <= 1.0 and 0.0 < r["online_hit_rate"] <= 1.0 and r["swaps"] > 0


def test_bulk_counts_match_oracle_and_per_layer_observation():
    """moe_cache_policy_observe_counts against the oracle on windows of several
    token steps; and for windows of one token step it equals observing each
    layer's routing in order (both libraries' plans compared with the oracle)."""
    L, E, S, k = 3, 24, 16, 3
    trace = synth.gen_routing_trace(12, L, E, k, 120, drift_every=30, drift_swaps=5)
    # windows of 1..7 token steps, counts summed per (layer, expert)
    bulk = native.CachePolicy(L, E, S, epoch=9, margin=1)
    orc = PolicyOracle(L, E, S, epoch=9, margin=1)
    slot_b = np.full((L, E), -1, np.int32)
    slot_o = [[-1] * E for _ in range(L)]
    rng = np.random.default_rng(3)
    t = 0
    while t < trace.shape[0]:
        w = int(rng.integers(1, 8))
        win = trace[t:t + w]
        counts = np.zeros((L, E), np.int32)
        for l in range(L):
            np.add.at(counts[l], win[:, l].ravel(), 1)
        bulk.observe_counts(counts, win.shape[0])
        orc.observe_counts(counts.tolist(), win.shape[0])
        assert bulk.plan(slot_b, 3) == orc.plan(slot_o, 3)
        np.testing.assert_array_equal(slot_b, np.array(slot_o, np.int32))
        t += w
    # one token step per window == per-layer observe
    per = native.CachePolicy(L, E, S, epoch=5, margin=0)
    one = native.CachePolicy(L, E, S, epoch=5, margin=0)
    s1 = np.full((L, E), -1, np.int32)
    s2 = np.full((L, E), -1, np.int32)
    for t in range(40):
        counts = np.zeros((L, E), np.int32)
        for l in range(L):
            per.observe(l, trace[t, l][None, :])
            np.add.at(counts[l], trace[t, l], 1)
        one.observe_counts(counts, 1)
        if t % 4 == 3:
            assert per.plan(s1, 5) == one.plan(s2, 5)
            np.testing.assert_array_equal(s1, s2)
