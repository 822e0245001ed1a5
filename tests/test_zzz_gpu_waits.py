"""Bounded in-kernel waits on the GPU: they give up with MOE_DEV_TIMEOUT
instead of hanging, and the context stays usable. (Kept in the last test file:
it runs after every parity test.)"""
import numpy as np
import pytest
import torch

from bit_expert_ffn_fp32_b200 import configs, native, synth
from bit_expert_ffn_fp32_b200.layer import MoEStack
from gpu_util import OUT_TOL, check_routing, oracle_layer, rel_err, run_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    return MoEStack(configs.TINY)


def test_bounded_waits_time_out_and_leave_the_context_usable(tiny):
    """The library's in-kernel waits on a counter that nothing raises and on an
    mbarrier phase that nothing completes give up after their 100 ms limit with
    MOE_DEV_TIMEOUT (no hang, no fault), and the context runs a layer after."""
    counter = torch.zeros(1, dtype=torch.int32, device="cuda")
    el = torch.zeros(2, dtype=torch.int64, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    native.debug_wait_probe(counter, 1, el, st)
    torch.cuda.synchronize()
    assert int(st.item()) & native.DEV_TIMEOUT
    e = el.cpu().numpy()
    assert np.all(e >= 90e6) and np.all(e < 10e9), e
    counter.fill_(3)                       # already at its target: no wait
    st.zero_()
    native.debug_wait_probe(counter, 3, el, st)
    torch.cuda.synchronize()
    assert int(el[0].item()) < 1e6 and int(st.item()) & native.DEV_TIMEOUT
    x = synth.gen_x(0, 0, configs.TINY.T, configs.TINY.d)
    b = run_layer(tiny, 0, x)
    ref = oracle_layer(tiny, 0, x)
    assert int(b.status.item()) == 0
    check_routing(b, ref, configs.TINY.T, configs.TINY.k, configs.TINY.E)
    assert rel_err(b.y[: configs.TINY.T].cpu().numpy().astype(np.float64), ref["y_partial"]) <= OUT_TOL
