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


def test_device_counts_equal_routing_and_drive_the_policy():
    """The decode kernels and the cache lookup add every routed pair to the
    device counters; after a window of token steps the counters equal the
    counts of the routing they returned, bit for bit, and the policy fed in bulk
    from them plans exactly what the oracle plans from the same counts."""
    import torch

    from policy import PolicyOracle

    wl = configs.STACK48.with_(layers=4, resident=64)
    stack = MoEStack(wl)
    L, E, k = wl.layers, wl.E, wl.k
    stack.expert_counts.zero_()
    host = np.zeros((L, E), np.int64)
    for step in range(5):      # one-layer launches and one stacked launch per step
        xs = np.stack([synth.gen_x(wl.seed, l, 2, wl.d, stream=3000 + step) for l in range(L)])
        if step % 2 == 0:
            for l in range(L):
                b = stack.forward_fused(l, torch.from_numpy(xs[l].view(np.int16)).cuda())
                torch.cuda.synchronize()
                np.add.at(host[l], b.idx[:2 * k].cpu().numpy(), 1)
        else:
            sb = stack.forward_stack(torch.from_numpy(xs.view(np.int16)).cuda())
            torch.cuda.synchronize()
            for l in range(L):
                np.add.at(host[l], sb.idx[l, :2 * k].cpu().numpy(), 1)
    x = synth.gen_x(wl.seed, 0, 40, wl.d, stream=3100)           # the step-by-step path (moe_cache_lookup)
    b = run_layer(stack, 0, x)
    np.add.at(host[0], b.idx[:40 * k].cpu().numpy(), 1)
    dev = stack.expert_counts.cpu().numpy()
    np.testing.assert_array_equal(dev, host)
    S = L * stack.R
    pol = native.CachePolicy(L, E, S, epoch=3, margin=1)
    orc = PolicyOracle(L, E, S, epoch=3, margin=1)
    pol.observe_counts(dev, 6)
    orc.observe_counts(dev.tolist(), 6)
    slot_l = np.stack(stack.slot_of_host).astype(np.int32)
    slot_o = slot_l.tolist()
    assert pol.plan(slot_l, 20) == orc.plan(slot_o, 20)


def test_swaps_overlap_running_layers_and_keep_parity():
    """A plan carried out asynchronously: the outgoing experts leave the slot
    tables on the layer stream, the incoming records (packed on the host) are
    copied into their slots on a side stream while layers keep running, and the
    new slots are committed after the copies. Layers run during the copies match
    the oracle with the outgoing experts as misses; layers after the commit
    match it with the incoming experts resident."""
    import torch

    wl = configs.STACK48.with_(layers=2, resident=64)
    stack = MoEStack(wl)
    L, E, k = wl.layers, wl.E, wl.k
    # a plan that swaps in experts routed by the probe tokens below
    probe = [synth.gen_x(wl.seed, l, 1, wl.d, stream=4000) for l in range(L)]
    swaps, slot_h = [], np.stack(stack.slot_of_host).astype(np.int32)
    for l in range(L):
        b = run_layer(stack, l, probe[l])
        ids = [int(e) for e in b.idx[:k].cpu().numpy()]
        missing = [e for e in ids if slot_h[l][e] < 0][:2]
        resident = [e for e in range(E) if slot_h[l][e] >= 0 and e not in ids][:len(missing)]
        for e_in, e_out in zip(missing, resident):
            swaps.append((int(slot_h[l][e_out]), l, e_in, l, e_out))
    assert swaps
    prepared = stack.prepare_swaps(swaps)
    side = torch.cuda.Stream()
    handle = stack.begin_swaps(prepared, side)
    during = []
    for rep in range(3):               # queued behind the unmapping, concurrent with the copies
        for l in range(L):
            x = synth.gen_x(wl.seed, l, 1, wl.d, stream=4100 + rep)
            during.append((l, x, _outputs(stack.forward_fused(l, torch.from_numpy(x.view(np.int16)).cuda()))))
    stack.commit_swaps(handle)
    torch.cuda.synchronize()
    outgoing = {(l, e_out) for _, l, _, _, e_out in swaps}
    incoming = {(l, e_in) for _, l, e_in, _, _ in swaps}
    slot_during = np.stack(stack.slot_of_host).astype(np.int32)
    for (l, e) in incoming:
        slot_during[l][e] = -1
    for l, x, out in during:
        ref = _oracle_with_slots(stack, l, x, slot_during[l])
        np.testing.assert_array_equal(out["sop"].cpu().numpy(), ref["slot_of_pair"])
        assert rel_err(out["y"].cpu().numpy().astype(np.float64), ref["y_partial"]) <= OUT_TOL
    for l in range(L):                 # after the commit: the probe tokens hit the incoming experts
        b = run_layer(stack, l, probe[l])
        ref = oracle_layer(stack, l, probe[l])
        check_routing(b, ref, 1, k, E)
        sop = b.sop[:k].cpu().numpy()
        ids = b.idx[:k].cpu().numpy()
        for j in range(k):
            if (l, int(ids[j])) in incoming:
                assert sop[j] >= 0
        assert rel_err(b.y[:1].cpu().numpy().astype(np.float64), ref["y_partial"]) <= OUT_TOL
    assert all(stack.slot_of_host[l][e] == -1 for l, e in outgoing)


def _outputs(b):
    return {"sop": b.sop[:b.T * 10].clone(), "y": b.y[:b.T].clone()}


def _oracle_with_slots(stack, layer, x, slot_row):
    import oracle as orc

    wl = stack.wl
    bias = None if stack.bias[layer] is None else stack.bias[layer].cpu().numpy()
    return orc.layer(x, synth.gen_router(stack.seed, layer, wl.E, wl.d), bias,
                     lambda e: stack.canonical_expert(layer, e), stack.canonical_expert(layer, wl.E), wl.k, wl.fmt,
                     slot_of=slot_row, layer_id=layer)
