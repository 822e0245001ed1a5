"""Prefill variants against the oracle: a pool holding both tiers (Q3 for the
most popular experts, Q2 for the rest), the 3-bit tier at prefill size, and a
prompt longer than one chunk run through the chunk loop (ragged last chunk).

The oracle is run on sampled token rows only: a token's logits, top-k, gates
and output depend on that token alone, so the oracle on the sampled rows gives
exactly the values of those rows in the full prompt. The permutation of the
full prompt is checked against a stable sort of the device's own top-k (the
definition of the counting sort), and the routed experts' output rows y_e
against the oracle's expert FFN at the first and the last pair of every
192-token tile of the experts sampled."""
import numpy as np
import pytest
import torch

from bit_expert_ffn_fp32_b200 import configs, synth
from bit_expert_ffn_fp32_b200.layer import MoEStack, x_tensor
from gpu_util import GATE_RTOL, OUT_TOL, full_check, oracle_layer, oracle_pair_rows, rel_err, run_layer

pytestmark = pytest.mark.gpu

MIXED = configs.WORKLOADS["prefill_T8192_d2048_E512_k10_f768_mixed_q3top128"]
Q3 = configs.WORKLOADS["prefill_T8192_d2048_E512_k10_f768_q3"]
CHUNKS = configs.WORKLOADS["prefill_chunks4_T32768_d2048_E512_k10_f768_q2"]


def _sample(T, n, seed):
    rng = np.random.default_rng(seed)
    return sorted(set([0, T - 1] + [int(t) for t in rng.choice(T, n, replace=False)]))


def _check_rows(stack, x, idx, w, logits, y, toks):
    """Routing and outputs of the sampled rows against the oracle on those rows."""
    ref = oracle_layer(stack, 0, x[toks])
    np.testing.assert_array_equal(logits[toks].view(np.uint32), ref["logit32"].view(np.uint32))
    np.testing.assert_array_equal(idx[toks], ref["idx"])
    np.testing.assert_allclose(w[toks], ref["gate"], rtol=GATE_RTOL, atol=1e-7)
    err = rel_err(y[toks].astype(np.float64), ref["y_partial"])
    assert err <= OUT_TOL, err
    return ref


def _perm_from_topk(idx, E):
    """Stable counting sort of the (t, j) pairs by expert id (numpy's stable sort)."""
    T, k = idx.shape
    order = np.argsort(idx.ravel(), kind="stable")
    counts = np.bincount(idx.ravel(), minlength=E)
    inv = np.empty(T * k, np.int64)
    inv[order] = np.arange(T * k)
    return {"counts": counts, "offsets": np.concatenate([[0], np.cumsum(counts)]), "sorted_tok": order // k,
            "sorted_j": order % k, "inv": inv}


def _check_layer(stack, x, experts_of_interest, seed):
    wl = stack.wl
    T, k, E = wl.T, wl.k, wl.E
    b = run_layer(stack, 0, x)
    assert int(b.status.item()) == 0
    idx = b.idx[:T * k].cpu().numpy().reshape(T, k)
    w = b.w[:T * k].cpu().numpy().reshape(T, k)
    logits = b.logits[:T].cpu().numpy()
    y = b.y[:T].cpu().numpy()
    _check_rows(stack, x, idx, w, logits, y, _sample(T, 40, seed))
    perm = _perm_from_topk(idx, E)
    for key, buf in (("counts", b.counts), ("offsets", b.offsets), ("sorted_tok", b.sorted_tok),
                     ("sorted_j", b.sorted_j), ("inv", b.inv)):
        n = perm[key].shape[0]
        np.testing.assert_array_equal(buf[:n].cpu().numpy(), perm[key], err_msg=key)
    counts, offs = perm["counts"], perm["offsets"]
    pos = set()
    for e in experts_of_interest(counts):
        for i0 in range(0, int(counts[e]), 192):
            pos.add(int(offs[e]) + i0)
            pos.add(int(offs[e]) + min(i0 + 192, int(counts[e])) - 1)
    pos = sorted(pos)
    assert pos
    want = oracle_pair_rows(stack, 0, x, perm, pos)
    got = b.y_perm[torch.tensor(pos, dtype=torch.long, device=b.y_perm.device)].cpu().numpy().astype(np.float64)
    expert_of = np.searchsorted(offs, np.array(pos), side="right") - 1
    worst = 0.0
    for e in np.unique(expert_of):
        sel = expert_of == e
        worst = max(worst, rel_err(got[sel], want[sel]))
    assert worst <= OUT_TOL, worst
    return b, perm


def test_mixed_pool_prefill():
    """Q3 for the 128 most popular experts, Q2 for the other 384 and the shared
    expert, in one pool: two expert calls (one per format) fill y_perm, the
    combine adds both. Sampled rows of every Q3 expert with tokens and of 40 Q2
    experts against the oracle dequantising each expert by its own format."""
    stack = MoEStack(MIXED)
    fmt = stack.fmt_of_host[0]
    assert (fmt == 3).sum() == 128 and (fmt == 2).sum() == 384
    x = synth.gen_x(0, 0, MIXED.T, MIXED.d, stream=31)

    def pick(counts):
        q3 = [e for e in range(MIXED.E) if fmt[e] == 3 and counts[e] > 0]
        q2 = [e for e in range(MIXED.E) if fmt[e] == 2 and counts[e] > 0]
        rng = np.random.default_rng(7)
        return q3 + [int(e) for e in rng.choice(q2, min(40, len(q2)), replace=False)]

    b, perm = _check_layer(stack, x, pick, 11)
    hot = perm["counts"][fmt == 3].sum()
    assert hot > perm["counts"][fmt == 2].sum()     # the Q3 tier carries most of the pairs


def test_q3_prefill_chunk():
    """The 3-bit tier at 8192 tokens: sampled rows, the permutation, and y_e at
    the tile ends of the 48 most loaded experts and 16 others."""
    stack = MoEStack(Q3)
    x = synth.gen_x(0, 0, Q3.T, Q3.d, stream=32)

    def pick(counts):
        order = np.argsort(-counts, kind="stable")
        rest = [int(e) for e in order[48:] if counts[e] > 0]
        rng = np.random.default_rng(8)
        return [int(e) for e in order[:48]] + [int(e) for e in rng.choice(rest, min(16, len(rest)), replace=False)]

    _check_layer(stack, x, pick, 12)


def test_chunk_loop_ragged_prompt():
    """A 17,384-token prompt in 8192-token chunks (8192, 8192, 1000): the loop's
    output equals each chunk run alone bit for bit, and sampled rows of every
    chunk (its first and last token among them) match the oracle."""
    wl = CHUNKS
    T = 2 * wl.chunk + 1000
    stack = MoEStack(wl)
    x = synth.gen_x(0, 0, T, wl.d, stream=33)
    xt = x_tensor(x)
    y = stack.forward_chunked(0, xt, wl.chunk)
    torch.cuda.synchronize()
    y = y.cpu().numpy()
    k = wl.k
    toks = []
    for c0 in range(0, T, wl.chunk):
        n = min(wl.chunk, T - c0)
        b = run_layer(stack, 0, x[c0:c0 + n])
        assert int(b.status.item()) == 0
        np.testing.assert_array_equal(y[c0:c0 + n], b.y[:n].cpu().numpy())
        toks += [c0 + t for t in _sample(n, 12, c0)]
        if c0 + n == T:
            idx = b.idx[:n * k].cpu().numpy().reshape(n, k)
            w = b.w[:n * k].cpu().numpy().reshape(n, k)
            logits = b.logits[:n].cpu().numpy()
            last = [t - c0 for t in toks if t >= c0]
            _check_rows(stack, x[c0:], idx, w, logits, y[c0:], last)
    ref = oracle_layer(stack, 0, x[toks])
    err = rel_err(y[toks].astype(np.float64), ref["y_partial"])
    assert err <= OUT_TOL, err


def test_chunk_loop_from_host_overlapped():
    """The pipelined host-to-host chunk loop (copies of the neighbouring chunks
    on side streams) gives the device chunk loop's output bit for bit, ragged
    last chunk included, and leaves nothing pending on the current stream's
    reader."""
    wl = CHUNKS
    T = 2 * wl.chunk + 1000
    stack = MoEStack(wl)
    x = synth.gen_x(0, 0, T, wl.d, stream=34)
    want = stack.forward_chunked(0, x_tensor(x), wl.chunk)
    torch.cuda.synchronize()
    x_host = torch.from_numpy(x.view(np.int16)).pin_memory()
    y_host = torch.full((T, wl.d), float("nan"), dtype=torch.float32).pin_memory()
    stack.forward_chunked_host(0, x_host, y_host, wl.chunk)
    torch.cuda.current_stream().synchronize()
    np.testing.assert_array_equal(y_host.numpy(), want.cpu().numpy())


# ---------------------------------------------------------------- Q3 on the tensor-core path
@pytest.fixture(scope="module")
def tiny_q3():
    return MoEStack(configs.TINY.with_(fmt=3))


@pytest.mark.parametrize("T", [128, 300, 777])
@pytest.mark.parametrize("combine", ["kernel", "atomic"])
def test_tc05_q3_tiny_shapes(tiny_q3, T, combine):
    """T*k >= 512 routes the Q3 expert calls to the tcgen05 grouped GEMMs
    (block-quad code units: d=512 is two quads, f=256 one): every token."""
    x = synth.gen_x(0, 0, T, configs.TINY.d, stream=1900 + T)
    full_check(tiny_q3, 0, x, combine=combine)


def test_tc05_q3_with_misses():
    """Q3 experts resident by Zipf rank (a quarter of them) at 600 tokens: the
    misses are left out of y on the tensor-core path too."""
    wl = configs.STACK48.with_(layers=1, T=600, fmt=3)
    stack = MoEStack(wl)
    x = synth.gen_x(0, 0, wl.T, wl.d, stream=1962)
    full_check(stack, 0, x, tokens=[0, 1, 299, 599])


def test_tc05_q3_every_pair_written_and_deterministic():
    """Every routed pair's y_e row is produced and two runs give identical bits."""
    wl = configs.VERIFY
    stack = MoEStack(wl)
    T = 1500
    x = x_tensor(synth.gen_x(0, 0, T, wl.d, stream=1951))
    b = stack.buffers(T)
    outs = []
    for fill in (12345.0, -777.0):
        b.y_perm.fill_(fill)
        b.h_ws.fill_(0xFF)
        stack.forward(0, x, b)
        torch.cuda.synchronize()
        assert int(b.status.item()) == 0
        yp = b.y_perm[:T * wl.k].clone()
        assert not bool(torch.isnan(yp).any())
        assert not bool((yp == fill).all(dim=1).any())
        outs.append(yp)
    assert torch.equal(outs[0], outs[1])
