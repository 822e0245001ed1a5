"""The allocation-free expert FFN call against the workspace one (GPU, C ABI).

moe_expert_ffn_q2_noalloc is for callers that cannot allocate device memory:
a plugin inside a host framework that owns all device buffers and passes the
plugin only its inputs and outputs, or a serving loop that allocates nothing
after start-up so that its memory use is fixed. The call keeps its scratch in
an array built into the library. These tests run it twice in a row, each time
on new tokens, and compare its output with moe_expert_ffn_q2 given a caller
workspace on the same routing; they also check that a request larger than the
built-in scratch is refused before anything runs. This file is collected last
so that a stop at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from bit_expert_ffn_fp32_b200 import configs, native, synth
from bit_expert_ffn_fp32_b200.layer import MoEStack, x_tensor

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3   # the layer-output tolerance used by every parity test


def _routed(stack, x, T):
    wl = stack.wl
    b = stack.buffers(T)
    b.status.zero_()
    native.route(x, stack.Wr[0], stack.bias[0], T, wl.d, wl.E, wl.k, b.logits, b.idx, b.w, b.status)
    native.permute(b.idx, T, wl.k, wl.E, b.counts, b.offsets, b.sorted_tok, b.sorted_j, b.inv, b.active, b.perm_ws,
                   0 if b.perm_ws is None else b.perm_ws.numel(), b.status)
    return b


_STACKS = {}


def _stack(wl):
    # one pool per workload for the whole file (building the 512-expert pool takes a while)
    if wl.name not in _STACKS:
        _STACKS[wl.name] = MoEStack(wl)
    return _STACKS[wl.name]


@pytest.mark.parametrize("wl,T", [(configs.TINY, 16), (configs.DECODE, 4), (configs.DECODE, 64)],
                         ids=["tiny_T16", "decode_T4", "decode_T64_tensor_core"])
def test_noalloc_matches_workspace_call_twice(wl, T):
    """T*k = 64 and 40 pairs run the weight-streaming kernels; 640 pairs (between
    512 and the 744-pair limit at d=2048, f=768) run the tensor-core GEMMs with
    h and the fp16 activation rows in the built-in array."""
    stack = _stack(wl)
    for call in range(2):
        x = x_tensor(synth.gen_x(wl.seed, 0, T, wl.d, stream=500 + call), stack.device)
        b = _routed(stack, x, T)
        n = T * wl.k
        y_ws = torch.full((n, wl.d), float("nan"), dtype=torch.float32, device=stack.device)
        y_na = torch.full((n, wl.d), float("nan"), dtype=torch.float32, device=stack.device)
        native.expert_ffn(stack.qpool, stack.slot_of[0], x, T, wl.d, wl.f, wl.E, wl.k, b.offsets, b.sorted_tok,
                          b.sorted_j, b.active, None, y_ws, b.h_ws, b.h_ws.numel(), b.status)
        native.expert_ffn_q2_noalloc(stack.qpool, stack.slot_of[0], x, T, wl.d, wl.f, wl.E, wl.k, b.offsets,
                                     b.sorted_tok, b.sorted_j, b.active, None, y_na, b.status)
        torch.cuda.synchronize()
        assert int(b.status.item()) == 0
        ref = y_ws.cpu().numpy().astype(np.float64)
        got = y_na.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(ref)) and np.all(np.isfinite(got))
        err = np.max(np.abs(got - ref)) / np.max(np.abs(ref))
        assert err <= OUT_TOL, (call, err)
        if T * wl.k >= 512:  # the tensor-core range also against the oracle, at every 16th sorted pair
            import oracle as orc
            from gpu_util import oracle_pair_rows

            x_bits = synth.gen_x(wl.seed, 0, T, wl.d, stream=500 + call)
            l32, _, _ = orc.router(x_bits, synth.gen_router(wl.seed, 0, wl.E, wl.d),
                                   None if stack.bias[0] is None else stack.bias[0].cpu().numpy())
            idx, _ = orc.topk(l32, wl.k)
            perm = orc.permute(idx, wl.E)
            np.testing.assert_array_equal(b.sorted_tok[:n].cpu().numpy(), perm["sorted_tok"])
            pos = sorted(set(range(0, n, 16)) | {n - 1})
            want = oracle_pair_rows(stack, 0, x_bits, perm, pos)
            err_o = np.max(np.abs(got[pos] - want)) / np.max(np.abs(want))
            assert err_o <= OUT_TOL, (call, err_o)


def test_noalloc_refuses_more_than_its_scratch():
    wl = configs.DECODE
    stack = MoEStack(wl.with_(E=16, k=4, resident=-1), layers=1)
    T = 2048                      # 2048 * 4 * 768 * 4 B = 24 MiB > 4 MiB
    dummy = torch.zeros(8, dtype=torch.int32, device="cuda")
    with pytest.raises(native.MoeError) as ei:
        native.expert_ffn_q2_noalloc(stack.qpool, dummy, dummy, T, wl.d, wl.f, 16, 4, dummy, dummy, dummy, dummy,
                                     None, dummy)
    assert ei.value.code == 3
