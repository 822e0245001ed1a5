"""CUDA path (through the C ABI) against the CPU oracle on the same seeded inputs.

Indices (router top-k, permutation, cache slots, miss list) must match bit for
bit, router logits too (the fp32 operation order is part of the definition);
gates within 1e-5 relative; layer outputs within max|y-y_ref|/max|y_ref| <= 2e-3.
"""
import numpy as np
import pytest
import torch

from bit_expert_ffn_fp32_b200 import configs, native, synth
from bit_expert_ffn_fp32_b200.layer import MoEStack, x_tensor
from gpu_util import OUT_TOL, check_routing, full_check, oracle_layer, oracle_pair_rows, rel_err, run_layer

pytestmark = pytest.mark.gpu


_full_check = full_check


@pytest.fixture(scope="module")
def tiny():
    return MoEStack(configs.TINY)


def test_tiny_layer(tiny):
    x = synth.gen_x(0, 0, configs.TINY.T, configs.TINY.d)
    _full_check(tiny, 0, x)


@pytest.mark.parametrize("T", [1, 2, 3, 5, 7, 8, 9, 13, 31, 64])
def test_tiny_ragged_token_counts(tiny, T):
    x = synth.gen_x(0, 0, T, configs.TINY.d, stream=100 + T)
    _full_check(tiny, 0, x)


def test_tiny_zero_tokens(tiny):
    b = tiny.buffers(0)
    x = torch.empty(0, configs.TINY.d, dtype=torch.int16, device="cuda")
    tiny.forward(0, x, b)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0 and int(b.active[0].item()) == 0 and int(b.miss_count.item()) == 0


def test_tiny_ties_zero_input(tiny):
    T = 3
    x = np.zeros((T, configs.TINY.d), np.uint16)
    b, ref, _ = _full_check(tiny, 0, x)
    np.testing.assert_array_equal(ref["idx"], np.tile(np.arange(configs.TINY.k), (T, 1)))
    assert np.all(b.y[:T].cpu().numpy() == 0)


@pytest.fixture(scope="module")
def decode():
    return MoEStack(configs.DECODE)


def test_decode_layer_full_size(decode):
    for s in range(3):
        x = synth.gen_x(0, 0, 1, configs.DECODE.d, stream=s)
        _full_check(decode, 0, x)


def test_decode_fused_gate_matches_combine(decode):
    """moe_expert_ffn with topk_w set (gate-weighted atomic accumulation) equals
    y_perm + moe_combine."""
    wl = configs.DECODE
    x = x_tensor(synth.gen_x(0, 0, 2, wl.d, stream=7))
    b = decode.buffers(2)
    decode.forward(0, x, b)
    y_ref = b.y[:2].clone()
    y2 = b.y_sh[:2].clone()
    native.expert_ffn(decode.qpool, decode.slot_of[0], x, 2, wl.d, wl.f, wl.E, wl.k, b.offsets, b.sorted_tok,
                      b.sorted_j, b.active, b.w, y2, b.h_ws, b.h_ws.numel(), b.status)
    torch.cuda.synchronize()
    assert rel_err(y2.cpu().numpy(), y_ref.cpu().numpy()) < 1e-5


@pytest.fixture(scope="module")
def verify():
    return MoEStack(configs.VERIFY)


def test_verify_layer_q3(verify):
    for s in range(2):
        x = synth.gen_x(0, 0, configs.VERIFY.T, configs.VERIFY.d, stream=s)
        _full_check(verify, 0, x)


def test_prefill_chunk_every_tile_against_the_oracle():
    """8192-token prefill chunk (tcgen05 grouped GEMMs). Routing, permutation and
    slots bit-exact for every token; y against the oracle at 64 tokens; and the
    routed experts' output rows y_e (before the gate) against the oracle's
    expert FFN at the first and the last pair of every (expert, 192-token N
    tile) of the persistent schedule, plus every pair of the most loaded expert."""
    wl = configs.PREFILL
    stack = MoEStack(wl)
    x = synth.gen_x(0, 0, wl.T, wl.d)
    rng = np.random.default_rng(0)
    toks = sorted(set([0, wl.T - 1] + [int(t) for t in rng.choice(wl.T, 62, replace=False)]))
    b, ref, err = _full_check(stack, 0, x, tokens=toks)
    assert len(toks) >= 64
    perm = ref["perm"]
    counts, offs = perm["counts"], perm["offsets"]
    assert counts.sum() == wl.T * wl.k and counts.max() > 500     # Zipf skew present
    tn = 192                                                      # tokens per N tile
    pos = set()
    for e in range(wl.E):
        for i0 in range(0, int(counts[e]), tn):
            pos.add(int(offs[e]) + i0)
            pos.add(int(offs[e]) + min(i0 + tn, int(counts[e])) - 1)
    big = int(np.argmax(counts))
    pos |= set(range(int(offs[big]), int(offs[big + 1])))
    pos = sorted(pos)
    want = oracle_pair_rows(stack, 0, x, perm, pos)
    got = b.y_perm[torch.tensor(pos, dtype=torch.long, device=b.y_perm.device)].cpu().numpy().astype(np.float64)
    pos_a = np.array(pos)
    expert_of = np.searchsorted(offs, pos_a, side="right") - 1
    worst = 0.0
    for e in np.unique(expert_of):
        sel = expert_of == e
        worst = max(worst, rel_err(got[sel], want[sel]))
    assert worst <= OUT_TOL, worst


def test_stack48_cache_and_misses():
    wl = configs.STACK48
    stack = MoEStack(wl)
    hits = total = 0
    for l in range(wl.layers):
        x = synth.gen_x(0, l, 1, wl.d)
        b = run_layer(stack, l, x)
        assert int(b.status.item()) == 0
        sample_y = l % 6 == 0
        ref = oracle_layer(stack, l, x, tokens=[0] if sample_y else [])
        check_routing(b, ref, 1, wl.k, wl.E)
        assert [m[:4] for m in stack.misses(b)] == [m[:4] for m in ref["misses"]]
        hits += int((b.sop[: wl.k].cpu().numpy() >= 0).sum())
        total += wl.k
        if sample_y:
            assert rel_err(b.y[:1].cpu().numpy().astype(np.float64), ref["y_partial"][:1]) <= OUT_TOL
            # the misses completed on the host give the full layer output
            y_full = _complete_on_host(stack, l, x, b)
            assert rel_err(y_full.astype(np.float64), ref["y_full"][:1]) <= OUT_TOL
    assert 0 < hits < total


def _complete_on_host(stack, layer, x_bits, b):
    """The GPU's partial y plus moe_complete_misses_host over the layer's miss
    list, the missed experts given in canonical host storage."""
    wl = stack.wl
    recs = np.array(stack.misses(b), dtype=[("layer", "<i4"), ("expert", "<i4"), ("token", "<i4"), ("j", "<i4"),
                                            ("gate", "<f4")])
    y = np.ascontiguousarray(b.y[: x_bits.shape[0]].cpu().numpy())
    if len(recs) == 0:
        return y
    canon = {e: stack.canonical_expert(layer, e) for e in sorted(set(recs["expert"].tolist()))}
    tab = native.expert_table(wl.E, canon)
    native.complete_misses_host(wl.fmt, wl.d, wl.f, tab, wl.E, recs, len(recs), layer, np.ascontiguousarray(x_bits),
                                x_bits.shape[0], y, 0)
    return y


# ---------------------------------------------------------------- device-side status
def test_bad_expert_id_is_flagged(tiny):
    wl = configs.TINY
    T, k, E = 4, wl.k, wl.E
    b = tiny.buffers(T)
    idx = torch.tensor([[0, 1, 2, 3], [4, 5, 6, 99], [7, 7, 8, 9], [1, 2, 3, 4]], dtype=torch.int32, device="cuda")
    b.status.zero_()
    native.permute(idx, T, k, E, b.counts, b.offsets, b.sorted_tok, b.sorted_j, b.inv, b.active, None, 0, b.status)
    torch.cuda.synchronize()
    assert int(b.status.item()) & native.DEV_BAD_INDEX


def test_bad_slot_and_miss_overflow(tiny):
    wl = configs.TINY
    T = 4
    x = x_tensor(synth.gen_x(0, 0, T, wl.d, stream=3))
    b = tiny.buffers(T)
    b.status.zero_()
    tiny.forward(0, x, b)
    slot_bad = tiny.slot_of[0].clone()
    slot_bad[:] = -1
    e0 = int(b.idx[0].item())
    slot_bad[e0] = tiny.num_slots + 5        # out of range: flagged, treated as a miss
    native.cache_lookup(slot_bad, tiny.num_slots, 0, b.idx, b.w, b.offsets, b.sorted_tok, b.sorted_j, T, wl.k, wl.E,
                        b.sop, b.miss, b.miss_count, 3, b.status)
    torch.cuda.synchronize()
    st = int(b.status.item())
    assert st & native.DEV_BAD_SLOT and st & native.DEV_MISS_OVERFLOW
    assert int(b.miss_count.item()) == T * wl.k
    assert np.all(b.sop[: T * wl.k].cpu().numpy() == -1)


def test_all_misses_gives_shared_only(tiny):
    wl = configs.TINY
    T = 5
    x_bits = synth.gen_x(0, 0, T, wl.d, stream=4)
    x = x_tensor(x_bits)
    b = tiny.buffers(T)
    saved = tiny.slot_of[0].clone()
    try:
        tiny.slot_of[0].fill_(-1)
        b.status.zero_()
        tiny.forward(0, x, b)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(b.y[:T].cpu().numpy(), b.y_sh[:T].cpu().numpy())
        assert int(b.miss_count.item()) == T * wl.k
    finally:
        tiny.slot_of[0].copy_(saved)


def test_multi_tile_permutation():
    # T spanning many 64-token tiles with a ragged last tile, compared with the oracle
    import oracle as orc
    wl = configs.TINY
    T, E, k = 1000, 64, 4
    rng = np.random.default_rng(5)
    idx_h = np.sort(np.stack([rng.choice(E, k, replace=False) for _ in range(T)]), axis=1).astype(np.int32)
    ref = orc.permute(idx_h, E)
    stack_b = MoEStack(wl.with_(T=T), layers=1)
    b = stack_b.buffers(T)
    idx = torch.from_numpy(idx_h.ravel()).cuda()
    b.status.zero_()
    native.permute(idx, T, k, E, b.counts, b.offsets, b.sorted_tok, b.sorted_j, b.inv, b.active, b.perm_ws,
                   b.perm_ws.numel(), b.status)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    for key, buf in (("counts", b.counts), ("offsets", b.offsets), ("sorted_tok", b.sorted_tok),
                     ("sorted_j", b.sorted_j), ("inv", b.inv)):
        np.testing.assert_array_equal(buf[: ref[key].shape[0]].cpu().numpy(), ref[key], err_msg=key)


# ---------------------------------------------------------------- router shapes
@pytest.mark.parametrize("T,d,E,k,ties", [
    (5, 256, 100, 7, False),      # few tokens: one warp per expert
    (64, 128, 200, 10, True),     # E not a multiple of the 32-expert tile, one 128-chunk
    (100, 384, 33, 4, False),     # ragged tokens and experts
    (300, 256, 512, 16, True),    # register top-k at its largest E, k = 16
    (97, 256, 600, 10, False),    # E > 512: the general top-k
])
def test_router_shapes(T, d, E, k, ties):
    """Logits bit for bit in the fixed fp32 order, selections exact, gates within
    1e-5, for token and expert counts that leave partial tiles; with ties, rows of
    Wr are duplicated so equal logits must resolve to the lower expert id."""
    import oracle as orc

    x_h = synth.gen_x(7, 0, T, d, stream=T + E)
    W_h = synth.gen_router(7, 0, E, d)
    if ties:
        W_h[E - 1] = W_h[3]
        W_h[11] = W_h[2]
    rng = np.random.default_rng(T * 1000 + E)
    bias_h = (rng.standard_normal(E) * 0.5).astype(np.float32)
    if ties:
        bias_h[E - 1], bias_h[11] = bias_h[3], bias_h[2]
    l32, _, _ = orc.router(x_h, W_h, bias_h)
    idx_ref, gate_ref = orc.topk(l32, k)
    x = torch.from_numpy(x_h.view(np.int16)).cuda()
    W = torch.from_numpy(W_h).cuda()
    bias = torch.from_numpy(bias_h).cuda()
    logits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    native.route(x, W, bias, T, d, E, k, logits, idx, w, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    np.testing.assert_array_equal(logits.cpu().numpy().view(np.uint32), l32.view(np.uint32))
    np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref)
    np.testing.assert_allclose(w.cpu().numpy(), gate_ref, rtol=1e-5, atol=1e-7)


# ---------------------------------------------------------------- tensor-core (prefill) path
@pytest.mark.parametrize("T", [256, 300, 777])
def test_tc05_path_tiny_shapes(tiny, T):
    """T*k >= 512 routes the Q2 expert calls to the tcgen05 grouped GEMMs
    (ragged N tiles, several M tiles, d=512 K loop)."""
    x = synth.gen_x(0, 0, T, configs.TINY.d, stream=900 + T)
    _full_check(tiny, 0, x)            # every token


def test_tc05_path_decode_shapes(decode):
    T = 1000
    x = synth.gen_x(0, 0, T, configs.DECODE.d, stream=950)
    _full_check(decode, 0, x, tokens=list(range(0, T, 61)) + [T - 1])


def test_tc05_every_pair_written_and_deterministic(decode):
    """Every routed pair's y_e row is produced (no tile skipped or doubled by the
    persistent schedule) and two runs give identical bits (no atomics in y_perm mode)."""
    wl = configs.DECODE
    T = 1500
    x = x_tensor(synth.gen_x(0, 0, T, wl.d, stream=951))
    b = decode.buffers(T)
    outs = []
    for fill in (12345.0, -777.0):
        b.y_perm.fill_(fill)
        b.h_ws.fill_(0xFF)            # NaN pattern in fp16 / fp32
        decode.forward(0, x, b)
        torch.cuda.synchronize()
        n = T * wl.k
        yp = b.y_perm[:n].clone()
        assert not bool(torch.isnan(yp).any())
        assert not bool((yp == fill).all(dim=1).any())
        outs.append(yp)
    assert torch.equal(outs[0], outs[1])


# ---------------------------------------------------------------- gate-weighted accumulation mode
@pytest.mark.parametrize("T", [5, 300])
def test_atomic_combine_tiny(tiny, T):
    """Shared expert written into y, routed experts added with gate-weighted
    atomics inside the expert call (mma.sync path at T=5, tcgen05 at T=300)."""
    x = synth.gen_x(0, 0, T, configs.TINY.d, stream=960 + T)
    _full_check(tiny, 0, x, combine="atomic")


def test_atomic_combine_decode_shapes(decode):
    T = 1000
    x = synth.gen_x(0, 0, T, configs.DECODE.d, stream=961)
    _full_check(decode, 0, x, tokens=list(range(0, T, 97)) + [T - 1], combine="atomic")


def test_atomic_combine_with_misses():
    """Residency by Zipf rank (stack workload shapes): misses are left out of y."""
    wl = configs.STACK48.with_(layers=1, T=600)
    stack = MoEStack(wl)
    x = synth.gen_x(0, 0, wl.T, wl.d, stream=962)
    b, ref, _ = _full_check(stack, 0, x, tokens=[0, 1, 299, 599], combine="atomic")
    assert 0 < int(b.miss_count.item()) < wl.T * wl.k
