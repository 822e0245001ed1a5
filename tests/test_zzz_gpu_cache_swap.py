"""The expert-cache policy driving the GPU pool: routing observed from a few
stacked decode layers feeds moe_cache_policy_*, its plans are carried out with
MoEStack.apply_swaps (records packed into their new slots, slot tables
updated), and the following layer calls still match the oracle under the new
slot tables: routing, hits and miss list bit for bit, output within 2e-3.
(Kept in a last test file: it runs after every parity test.)"""
import numpy as np
import pytest

from bit_expert_ffn_fp32_b200 import configs, native, synth
from bit_expert_ffn_fp32_b200.layer import MoEStack
from gpu_util import OUT_TOL, check_routing, oracle_layer, rel_err, run_layer

pytestmark = pytest.mark.gpu


def test_policy_swaps_into_the_gpu_pool_keep_parity():
    wl = configs.STACK48.with_(layers=3, resident=64)
    stack = MoEStack(wl)
    L, E, k = wl.layers, wl.E, wl.k
    S = L * stack.R
    pol = native.CachePolicy(L, E, S, epoch=64, margin=0)
    slot = np.stack(stack.slot_of_host).astype(np.int32)
    swapped = 0
    for step in range(6):
        for l in range(L):
            x = synth.gen_x(wl.seed, l, 1, wl.d, stream=1000 + step)
            b = run_layer(stack, l, x)
            assert int(b.status.item()) == 0
            pol.observe(l, b.idx[:k].cpu().numpy().reshape(1, k))
        swaps = pol.plan(slot, 12)
        stack.apply_swaps(swaps)
        swapped += len(swaps)
        np.testing.assert_array_equal(slot, np.stack(stack.slot_of_host))
        held = slot[slot >= 0]
        assert len(set(held.tolist())) == len(held) <= S
    assert swapped > 0
    for l in range(L):
        x = synth.gen_x(wl.seed, l, 1, wl.d, stream=2000)
        b = run_layer(stack, l, x)
        ref = oracle_layer(stack, l, x, tokens=[0])
        assert int(b.status.item()) == 0
        check_routing(b, ref, 1, k, E)
        assert [m[:4] for m in stack.misses(b)] == [m[:4] for m in ref["misses"]]
        assert rel_err(b.y[:1].cpu().numpy().astype(np.float64), ref["y_partial"][:1]) <= OUT_TOL
