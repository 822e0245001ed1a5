"""The one-launch decode layer (moe_layer_decode) against the CPU oracle and
against the step-by-step calls (GPU, C ABI).

Routing, permutation, cache slots and misses must be bit-exact; y within
max|y-y_ref|/max|y_ref| <= 2e-3 of the oracle.
"""
import numpy as np
import pytest
import torch

from bit_expert_ffn_fp32_b200 import configs, native, synth
from bit_expert_ffn_fp32_b200.layer import MoEStack, x_tensor
from gpu_util import OUT_TOL, check_routing, oracle_layer, rel_err

pytestmark = pytest.mark.gpu


def _fused(stack, layer, x_bits):
    x = x_tensor(x_bits, stack.device)
    b = stack.buffers(x.shape[0])
    b.status.zero_()
    b.y.fill_(float("nan"))
    stack.forward_fused(layer, x, b)
    torch.cuda.synchronize()
    return b


def _check(stack, layer, x_bits):
    wl = stack.wl
    T = x_bits.shape[0]
    b = _fused(stack, layer, x_bits)
    assert int(b.status.item()) == 0
    ref = oracle_layer(stack, layer, x_bits)
    check_routing(b, ref, T, wl.k, wl.E)
    assert [m[:4] for m in stack.misses(b)] == [m[:4] for m in ref["misses"]]
    assert int(b.miss_count.item()) == ref["miss_count"]
    err = rel_err(b.y[:T].cpu().numpy().astype(np.float64), ref["y_partial"])
    assert err <= OUT_TOL, err
    return b, ref


@pytest.fixture(scope="module")
def tiny():
    return MoEStack(configs.TINY)


@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 7, 8])
def test_fused_tiny_token_counts(tiny, T):
    _check(tiny, 0, synth.gen_x(0, 0, T, configs.TINY.d, stream=300 + T))


def test_fused_tiny_ties(tiny):
    b, ref = _check(tiny, 0, np.zeros((3, configs.TINY.d), np.uint16))
    assert np.all(b.y[:3].cpu().numpy() == 0)


@pytest.fixture(scope="module")
def decode():
    return MoEStack(configs.DECODE)


def test_fused_decode_layer(decode):
    for s in range(3):
        _check(decode, 0, synth.gen_x(0, 0, 1, configs.DECODE.d, stream=s))


def test_fused_equals_separate_calls(decode):
    wl = configs.DECODE
    for T in (1, 4, 8):
        x_bits = synth.gen_x(0, 0, T, wl.d, stream=40 + T)
        x = x_tensor(x_bits)
        b = decode.buffers(T)
        decode.forward(0, x, b)
        torch.cuda.synchronize()
        sep = {k: getattr(b, k)[: T * wl.k].clone() for k in ("idx", "w", "sorted_tok", "sorted_j", "inv", "sop")}
        y_sep = b.y[:T].clone()
        b2 = _fused(decode, 0, x_bits)
        for k, v in sep.items():
            assert torch.equal(getattr(b2, k)[: T * wl.k], v), k
        assert rel_err(b2.y[:T].cpu().numpy(), y_sep.cpu().numpy()) < 1e-5


def test_fused_repeated_launches_reset_counters(decode):
    wl = configs.DECODE
    x = x_tensor(synth.gen_x(0, 0, 2, wl.d, stream=77))
    b = decode.buffers(2)
    b.status.zero_()
    ys = []
    for _ in range(50):
        decode.forward_fused(0, x, b, outputs=False)
        ys.append(b.y[:2].clone())
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    ws = decode.decode_workspace(2)
    assert int(ws[:8].view(torch.int32).abs().sum().item()) == 0     # barrier counters back at zero
    for y in ys[1:]:
        assert rel_err(y.cpu().numpy(), ys[0].cpu().numpy()) < 1e-5


@pytest.fixture(scope="module")
def verify():
    return MoEStack(configs.VERIFY)


def test_fused_verify_q3(verify):
    for s in range(2):
        _check(verify, 0, synth.gen_x(0, 0, 4, configs.VERIFY.d, stream=s))


@pytest.mark.parametrize("T", [2, 8])
def test_fused_verify_q3_wider_batches(verify, T):
    """MTP verify batches of one token plus 1 or 7 drafts on Q3 experts."""
    for s in range(2):
        _check(verify, 0, synth.gen_x(0, 0, T, configs.VERIFY.d, stream=700 + 10 * T + s))


@pytest.mark.parametrize("T", [2, 4, 8])
def test_fused_decode_q2_batches(decode, T):
    """Q2 layer with 2, 4 and 8 tokens (several tokens per expert), against the oracle."""
    for s in range(2):
        _check(decode, 0, synth.gen_x(0, 0, T, configs.DECODE.d, stream=800 + 10 * T + s))


def test_fused_with_misses():
    wl = configs.STACK48
    stack = MoEStack(wl, layers=3)
    for l in range(3):
        b, ref = _check(stack, l, synth.gen_x(0, l, 1, wl.d))
    # all experts missing: y is the shared expert alone
    x_bits = synth.gen_x(0, 0, 2, wl.d, stream=9)
    saved = stack.slot_of[0].clone()
    try:
        stack.slot_of[0].fill_(-1)
        b = _fused(stack, 0, x_bits)
        y_sh = b.y[:2].clone()
        assert int(b.miss_count.item()) == 2 * wl.k
        stack.forward(0, x_tensor(x_bits), b)
        torch.cuda.synchronize()
        # the same fp32 sums in another association (the fused kernel adds each block's
        # four MMA partials after the fact; the step-by-step kernels chain them)
        assert rel_err(y_sh.cpu().numpy(), b.y_sh[:2].cpu().numpy()) < 1e-5
    finally:
        stack.slot_of[0].copy_(saved)


def test_stacked_layers_one_launch():
    """moe_stack_decode over 6 layers of the 48-layer workload (25% resident):
    every layer's routing, slots and misses bit-exact and y within 2e-3 of the
    oracle, and equal to the one-layer call on the same layer."""
    wl = configs.STACK48
    L = 6
    stack = MoEStack(wl, layers=L)
    xs = np.stack([synth.gen_x(0, l, 2, wl.d, stream=900) for l in range(L)])
    x = torch.from_numpy(xs.view(np.int16)).cuda()
    b = stack.stack_buffers(2)
    b.status.zero_()
    b.y.fill_(float("nan"))
    stack.forward_stack(x, b)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    ws = stack.decode_workspace(2)
    assert int(ws[:8].view(torch.int32).abs().sum().item()) == 0
    n = 2 * wl.k
    for l in range(L):
        ref = oracle_layer(stack, l, xs[l])
        np.testing.assert_array_equal(b.idx[l, :n].cpu().numpy().reshape(2, wl.k), ref["idx"])
        np.testing.assert_allclose(b.w[l, :n].cpu().numpy().reshape(2, wl.k), ref["gate"], rtol=1e-5, atol=1e-7)
        np.testing.assert_array_equal(b.sop[l, :n].cpu().numpy(), ref["slot_of_pair"])
        assert [m[:4] for m in stack.stack_misses(b, l)] == [m[:4] for m in ref["misses"]]
        assert int(b.miss_count[l].item()) == ref["miss_count"]
        err = rel_err(b.y[l, :2].cpu().numpy().astype(np.float64), ref["y_partial"])
        assert err <= OUT_TOL, (l, err)
        one = _fused(stack, l, xs[l])
        assert rel_err(b.y[l, :2].cpu().numpy(), one.y[:2].cpu().numpy()) < 1e-5


def test_stacked_layers_host_misses_overlapped():
    """The stacked launch writes each layer's miss list into mapped pinned host
    memory (count last); the miss engine, given the layers before the launch
    has finished, completes them on host threads while the GPU runs. GPU y plus
    the engine's sums must equal the oracle's full layer output (misses
    included) within 2e-3, and the published lists the oracle's."""
    from bit_expert_ffn_fp32_b200.layer import MISS_DTYPE

    wl = configs.STACK48
    L, T = 6, 1
    stack = MoEStack(wl, layers=L)
    xs = np.stack([synth.gen_x(0, l, T, wl.d, stream=901) for l in range(L)])
    x = torch.from_numpy(xs.view(np.int16)).cuda()
    b0 = stack.stack_buffers(T)        # a first pass tells which experts miss
    stack.forward_stack(x, b0)
    torch.cuda.synchronize()
    missed = [sorted(set(m[1] for m in stack.stack_misses(b0, l))) for l in range(L)]
    assert sum(len(m) for m in missed) > 0
    canon = [{e: stack.canonical_expert(l, e) for e in missed[l]} for l in range(L)]
    tabs = [native.expert_table(wl.E, c) for c in canon]
    b = stack.stack_buffers(T, host_misses=True)
    cap = b.idx.shape[1]
    cnt = b.miss_count.view(np.int32)
    miss_h = b.miss.view(MISS_DTYPE, (L, cap))
    y_add = np.zeros((L, T, wl.d), np.float32)
    eng = native.MissEngine(0)
    try:
        cnt[:] = -1
        b.status.zero_()
        stack.forward_stack(x, b)
        for l in range(L):
            eng.submit(wl.fmt, wl.d, wl.f, tabs[l], wl.E, miss_h[l], cnt[l:l + 1], cap, l,
                       np.ascontiguousarray(xs[l]), T, y_add[l])
        eng.wait()
    finally:
        eng.close()
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    y_full = b.y[:, :T].cpu().numpy().astype(np.float64) + y_add
    for l in range(L):
        ref = oracle_layer(stack, l, xs[l])
        assert [tuple(r)[:4] for r in miss_h[l, : int(cnt[l])]] == [m[:4] for m in ref["misses"]]
        err = rel_err(y_full[l], ref["y_full"])
        assert err <= OUT_TOL, (l, err)


def test_fused_rejects_unsupported(tiny):
    wl = configs.TINY
    x = torch.zeros(9, wl.d, dtype=torch.int16, device="cuda")
    with pytest.raises(native.MoeError) as ei:
        native.layer_decode(tiny.qpool, tiny.slot_of[0], tiny.num_slots - 1, 0, x, tiny.Wr[0], None, 9, wl.d, wl.f,
                            wl.E, wl.k, y=torch.empty(9, wl.d, device="cuda"), ws=tiny.decode_workspace(1),
                            ws_bytes=tiny.decode_workspace(1).numel())
    assert ei.value.code == 2


@pytest.mark.parametrize("T", [1, 2, 4])
def test_fused_all_logits_equal(decode, T):
    """x = 0 and no bias: all 512 logits tie, so far more than 64 keys reach the
    selection threshold and the exact per-warp path runs; the experts must be
    0..k-1 (ties go to the lower id) with equal gates."""
    wl = configs.DECODE
    saved = decode.bias[0].clone()
    try:
        decode.bias[0].zero_()
        b, ref = _check(decode, 0, np.zeros((T, wl.d), np.uint16))
        np.testing.assert_array_equal(ref["idx"], np.tile(np.arange(wl.k), (T, 1)))
    finally:
        decode.bias[0].copy_(saved)


@pytest.mark.parametrize("T", [1, 2])
def test_fused_many_candidates_fallback(decode, T):
    """Experts in 10 of the 32 lanes (id % 32 < 10) all outrank the rest, so more
    than 64 candidates clear the selection threshold and the round-based path runs."""
    wl = configs.DECODE
    saved = decode.bias[0].clone()
    try:
        boost = torch.zeros_like(saved)
        boost[(torch.arange(wl.E, device=saved.device) % 32) < 10] = 100.0
        decode.bias[0].copy_(saved + boost)
        for s in range(2):
            _check(decode, 0, synth.gen_x(0, 0, T, wl.d, stream=600 + s))
    finally:
        decode.bias[0].copy_(saved)
