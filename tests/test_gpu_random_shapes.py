"""Randomised shapes through the CUDA path against the oracle (hypothesis, a
fixed derandomised sample so every run checks the same cases).

Each example draws a layer -- code format (Q2, Q3 or a pool holding both), d,
f, E, k, T, router bias on or off, the fraction of experts resident -- builds
its pool, and runs the step-by-step calls (T*k >= 512 reaches the tensor-core
GEMMs) and, for T <= 8, the one-launch layer. Routing, permutation, slots and
the miss list must match the oracle bit for bit, y within 2e-3 at every token."""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings, strategies as st

from bit_expert_ffn_fp32_b200 import configs, synth
from bit_expert_ffn_fp32_b200.layer import MoEStack, x_tensor
from gpu_util import OUT_TOL, check_routing, full_check, oracle_layer, rel_err

pytestmark = pytest.mark.gpu

SETTINGS = dict(deadline=None, derandomize=True, database=None,
                suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])


@st.composite
def layers(draw, max_T):
    fmt = draw(st.sampled_from([2, 3, 23]))          # 23: both tiers in one pool
    d = draw(st.sampled_from([256, 512, 1024]))
    f = draw(st.sampled_from([256, 512, 768]))
    E = draw(st.integers(2, 256))
    k = draw(st.integers(1, min(16, E)))
    T = draw(max_T(k))
    zipf = draw(st.booleans())
    resident = draw(st.sampled_from([-1, -1, max(1, E // 4), max(1, E // 2)]))
    seed = draw(st.integers(0, 2**16))
    q3_top = max(1, E // 3) if fmt == 23 else 0
    name = f"rand_T{T}_d{d}_E{E}_k{k}_f{f}_fmt{fmt}_z{int(zipf)}_r{resident}_s{seed}"
    return configs.Workload(name, T, d, E, k, f, 2 if fmt == 23 else fmt, zipf=zipf, resident=resident,
                            seed=seed, q3_top=q3_top)


def _step_T(k):
    # small batches, and batches whose T*k reaches the tensor-core path
    return st.one_of(st.integers(1, 40), st.integers((512 + k - 1) // k, (512 + k - 1) // k + 90))


@settings(max_examples=24, **SETTINGS)
@given(layers(_step_T))
def test_random_layers_step_path(wl):
    stack = MoEStack(wl)
    x = synth.gen_x(wl.seed, 0, wl.T, wl.d, stream=7)
    full_check(stack, 0, x)


@settings(max_examples=20, **SETTINGS)
@given(layers(lambda k: st.integers(1, 8)))
def test_random_layers_one_launch(wl):
    if wl.q3_top:                       # the one-launch layer reads a single-format pool
        wl = wl.with_(q3_top=0)
    stack = MoEStack(wl)
    x = synth.gen_x(wl.seed, 0, wl.T, wl.d, stream=8)
    xt = x_tensor(x, stack.device)
    b = stack.buffers(wl.T)
    b.status.zero_()
    stack.forward_fused(0, xt, b)
    import torch

    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    ref = oracle_layer(stack, 0, x)
    check_routing(b, ref, wl.T, wl.k, wl.E)
    assert [m[:4] for m in stack.misses(b)] == [m[:4] for m in ref["misses"]]
    err = rel_err(b.y[:wl.T].cpu().numpy().astype(np.float64), ref["y_partial"])
    assert err <= OUT_TOL, err
