"""Shared helpers for the GPU parity tests (CUDA path vs the CPU oracle)."""
from __future__ import annotations

import numpy as np
import torch

import oracle as orc
from bit_expert_ffn_fp32_b200 import synth
from bit_expert_ffn_fp32_b200.layer import MoEStack, x_tensor

OUT_TOL = 2e-3      # max|y - y_ref| / max|y_ref| per layer
GATE_RTOL = 1e-5


def run_layer(stack: MoEStack, layer: int, x_bits: np.ndarray, combine: str = "kernel"):
    x = x_tensor(x_bits, stack.device)
    b = stack.buffers(x.shape[0])
    b.status.zero_()
    stack.forward(layer, x, b, combine=combine)
    torch.cuda.synchronize()
    return b


def oracle_layer(stack: MoEStack, layer: int, x_bits: np.ndarray, tokens=None):
    wl = stack.wl
    Wr = stack.Wr[layer].cpu().numpy()
    bias = None if stack.bias[layer] is None else stack.bias[layer].cpu().numpy()
    # inputs regenerated from the seeded generator, never read back from the device
    Wr_gen = synth.gen_router(stack.seed, layer, wl.E, wl.d)
    assert np.array_equal(Wr, Wr_gen)
    return orc.layer(x_bits, Wr_gen, bias, lambda e: stack.canonical_expert(layer, e),
                     stack.canonical_expert(layer, wl.E), wl.k, wl.fmt, slot_of=stack.slot_of_host[layer],
                     layer_id=layer, tokens=tokens, fmt_of=stack.fmt_of_host[layer] if stack.mixed else None)


def rel_err(y: np.ndarray, ref: np.ndarray) -> float:
    return float(np.max(np.abs(y - ref)) / max(np.max(np.abs(ref)), 1e-30))


def check_routing(b, ref, T: int, k: int, E: int):
    logits = b.logits[:T].cpu().numpy()
    np.testing.assert_array_equal(logits.view(np.uint32), ref["logit32"].view(np.uint32))
    idx = b.idx[: T * k].cpu().numpy().reshape(T, k)
    np.testing.assert_array_equal(idx, ref["idx"])
    w = b.w[: T * k].cpu().numpy().reshape(T, k)
    np.testing.assert_allclose(w, ref["gate"], rtol=GATE_RTOL, atol=1e-7)
    p = ref["perm"]
    for key, buf in (("counts", b.counts), ("offsets", b.offsets), ("sorted_tok", b.sorted_tok),
                     ("sorted_j", b.sorted_j), ("inv", b.inv)):
        n = p[key].shape[0]
        np.testing.assert_array_equal(buf[:n].cpu().numpy(), p[key], err_msg=key)
    na = int(p["active"][0])
    np.testing.assert_array_equal(b.active[: na + 1].cpu().numpy(), p["active"][: na + 1])
    np.testing.assert_array_equal(b.sop[: T * k].cpu().numpy(), ref["slot_of_pair"])


def oracle_pair_rows(stack: MoEStack, layer: int, x_bits: np.ndarray, perm: dict, positions) -> np.ndarray:
    """The oracle's y_e row (expert output before the gate) of every sorted pair
    position in `positions`, from the oracle's own permutation `perm`; each
    expert is dequantised once (fp64 [len(positions)][d])."""
    wl = stack.wl
    xf = orc.bf16_to_f64(x_bits)
    offs = perm["offsets"]
    positions = list(positions)
    out = np.empty((len(positions), wl.d), np.float64)
    by_e: dict[int, list[int]] = {}
    for i, s in enumerate(positions):
        e = int(np.searchsorted(offs, s, side="right") - 1)
        by_e.setdefault(e, []).append(i)
    for e, rows in by_e.items():
        W = orc.dequant_expert(stack.canonical_expert(layer, e), stack.expert_fmt(layer, e))
        toks = [int(perm["sorted_tok"][positions[i]]) for i in rows]
        out[rows] = orc.expert_ffn(W, xf[toks])
    return out


def full_check(stack, layer, x_bits, tokens=None, combine="kernel"):
    """One forward() against the oracle: routing, permutation, slots and the
    miss list bit for bit, y within OUT_TOL at `tokens` (default every token)."""
    wl = stack.wl
    T = x_bits.shape[0]
    b = run_layer(stack, layer, x_bits, combine)
    ref = oracle_layer(stack, layer, x_bits, tokens=tokens)
    assert int(b.status.item()) == 0
    check_routing(b, ref, T, wl.k, wl.E)
    misses = stack.misses(b)
    assert [m[:4] for m in misses] == [m[:4] for m in ref["misses"]]
    assert int(b.miss_count.item()) == ref["miss_count"]
    toks = ref["tokens"]
    y = b.y[:T].cpu().numpy().astype(np.float64)
    err = rel_err(y[toks], ref["y_partial"][toks])
    assert err <= OUT_TOL, err
    return b, ref, err
