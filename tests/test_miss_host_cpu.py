"""Host completion of the miss list (moe_complete_misses_host) against the oracle.

The library computes the missed experts on the host from their canonical
storage (lookup-table dot products per 64-block); the oracle computes the same
SwiGLU experts in fp64 from the dequantised weights. Every record adds
gate * FFN_e(x_t) into y[t]; y is compared with y0 + the sum of the oracle's
terms, within max|y - y_ref| / max|y_ref| <= 1e-5 (fp32 against fp64).
"""
import ctypes as C

import numpy as np
import pytest

from bit_expert_ffn_fp32_b200 import native, synth

MISS_DT = np.dtype([("layer", "<i4"), ("expert", "<i4"), ("token", "<i4"), ("j", "<i4"), ("gate", "<f4")])
TOL = 1e-5


def _experts(fmt, d, f, ids, seed=11, layer=0):
    return {e: synth.gen_expert(seed, layer, e, fmt, d, f) for e in ids}


def _oracle_terms(orc, canon, fmt, x_bits, records):
    xf = orc.bf16_to_f64(x_bits)
    memo = {}
    out = np.zeros((x_bits.shape[0], x_bits.shape[1]), np.float64)
    for r in records:
        e = int(r["expert"])
        if e not in memo:
            memo[e] = orc.dequant_expert(canon[e], fmt)
        out[int(r["token"])] += float(r["gate"]) * orc.expert_ffn(memo[e], xf[int(r["token"])])[0]
    return out


@pytest.mark.parametrize("fmt", [2, 3])
@pytest.mark.parametrize("nthreads", [1, 3])
def test_complete_misses_matches_oracle(orc, fmt, nthreads):
    d, f, E, T = 512, 256, 6, 5
    canon = _experts(fmt, d, f, range(E))
    tab = native.expert_table(E, canon)
    x = synth.gen_x(3, 0, T, d, stream=7)
    # two misses on one token, two tokens on one expert
    recs = np.array([(0, 4, 0, 2, 0.30), (0, 1, 3, 0, 0.05), (0, 4, 2, 7, 0.125), (0, 0, 0, 5, 0.2),
                     (0, 5, 4, 1, 0.9)], MISS_DT)
    y0 = np.random.default_rng(2).standard_normal((T, d)).astype(np.float32)
    y = y0.copy()
    native.complete_misses_host(fmt, d, f, tab, E, recs, len(recs), 0, x, T, y, nthreads)
    ref = y0.astype(np.float64) + _oracle_terms(orc, canon, fmt, x, recs)
    err = np.max(np.abs(y - ref)) / np.max(np.abs(ref))
    assert err <= TOL, err
    untouched = [t for t in range(T) if t not in set(recs["token"].tolist())]
    np.testing.assert_array_equal(y[untouched], y0[untouched])


@pytest.mark.parametrize("fmt", [2, 3])
def test_complete_misses_full_size_and_thread_independence(orc, fmt):
    """d=2048, f=768 (the decode shapes); only the named experts are given;
    the result is the same bit for bit for 1 and 4 threads."""
    d, f, E, T = 2048, 768, 512, 3
    canon = _experts(fmt, d, f, [17, 300], seed=5)
    tab = native.expert_table(E, canon)
    x = synth.gen_x(5, 0, T, d, stream=1)
    recs = np.array([(0, 300, 2, 3, 0.4), (0, 17, 0, 0, 0.6), (0, 300, 0, 9, 0.25)], MISS_DT)
    ys = []
    for nth in (1, 4):
        y = np.zeros((T, d), np.float32)
        native.complete_misses_host(fmt, d, f, tab, E, recs, len(recs), 0, x, T, y, nth)
        ys.append(y)
    np.testing.assert_array_equal(ys[0], ys[1])
    ref = _oracle_terms(orc, canon, fmt, x, recs)
    err = np.max(np.abs(ys[0] - ref)) / np.max(np.abs(ref))
    assert err <= TOL, err
    assert np.all(ys[0][1] == 0)


def test_complete_misses_special_blocks(orc):
    """Blocks with scale 0 (w = m, the block sum path alone), all-zero codes
    with min 0 (contributes nothing), and power-of-two scales."""
    d, f, E, T = 256, 256, 1, 1
    ex = synth.gen_expert(9, 0, 0, 2, d, f)
    for m in ("gate", "up", "down"):
        ex[m]["scale"][:, ::3] = 0                      # s = 0: w = m
        ex[m]["codes"][::2, :] = 0
        ex[m]["min"][::2, :] = 0                        # rows with w = 0 where s = 0 too
        ex[m]["scale"][:, 1::3] = 0x3800                # 0.5
    tab = native.expert_table(E, {0: ex})
    x = synth.gen_x(2, 0, T, d)
    recs = np.array([(3, 0, 0, 0, 1.0)], MISS_DT)
    y = np.zeros((T, d), np.float32)
    native.complete_misses_host(2, d, f, tab, E, recs, 1, 3, x, T, y, 1)
    ref = _oracle_terms(orc, {0: ex}, 2, x, recs)
    assert np.max(np.abs(y - ref)) / np.max(np.abs(ref)) <= TOL


def test_complete_misses_rejects_bad_records_before_writing():
    d, f, E, T = 512, 256, 3, 2
    canon = _experts(2, d, f, [0, 1])  # expert 2 is not given
    tab = native.expert_table(E, canon)
    x = synth.gen_x(1, 0, T, d)
    y = np.ones((T, d), np.float32)
    L = native.lib

    def call(recs, fmt=2):
        return L.moe_complete_misses_host(fmt, d, f, C.cast(tab, C.c_void_p), E, recs.ctypes.data, len(recs), 0,
                                          x.ctypes.data, T, y.ctypes.data, 1)

    good = (0, 1, 1, 0, 0.5)
    for bad in [(1, 1, 1, 0, 0.5),    # another layer
                (0, 3, 1, 0, 0.5),    # expert outside [0, E)
                (0, -1, 1, 0, 0.5),
                (0, 1, 2, 0, 0.5),    # token outside [0, T)
                (0, 2, 0, 0, 0.5)]:   # expert whose matrices are not given
        assert call(np.array([good, bad], MISS_DT)) == 1
        assert np.all(y == 1.0)
    # Q3 needs the high-bit plane, which Q2 storage lacks
    assert call(np.array([good], MISS_DT), fmt=3) == 1
    assert np.all(y == 1.0)
    assert call(np.zeros(0, MISS_DT)) == 0
    assert np.all(y == 1.0)


# ---------------------------------------------------------------- miss engine
def test_miss_engine_matches_blocking_call_as_counts_are_published():
    """Layers submitted before their records exist: each count starts at -1 and
    another thread fills the records and then the count (as the GPU does
    through mapped memory), layer by layer. The engine's y equals the blocking
    moe_complete_misses_host result bit for bit."""
    import threading
    import time

    d, f, E, T, L = 512, 256, 8, 4, 5
    fmt = 2
    canons = [_experts(fmt, d, f, range(E), seed=20 + l, layer=l) for l in range(L)]
    tabs = [native.expert_table(E, c) for c in canons]
    xs = [synth.gen_x(4, l, T, d, stream=2) for l in range(L)]
    rng = np.random.default_rng(8)
    recs = []
    for l in range(L):
        n = int(rng.integers(1, 7))
        recs.append(np.array([(l, int(rng.integers(0, E)), int(rng.integers(0, T)), j, float(rng.random()))
                              for j in range(n)], MISS_DT))
    cap = 8
    miss_bufs = [np.zeros(cap, MISS_DT) for _ in range(L)]
    counts = np.full(L, -1, np.int32)
    ys = [np.zeros((T, d), np.float32) for _ in range(L)]
    eng = native.MissEngine(3)
    try:
        for l in range(L):
            eng.submit(fmt, d, f, tabs[l], E, miss_bufs[l], counts[l:l + 1], cap, l, xs[l], T, ys[l])

        def publish():
            for l in range(L):
                time.sleep(0.02)
                miss_bufs[l][: len(recs[l])] = recs[l]
                counts[l] = len(recs[l])

        th = threading.Thread(target=publish)
        th.start()
        eng.wait()
        th.join()
    finally:
        eng.close()
    for l in range(L):
        ref = np.zeros((T, d), np.float32)
        native.complete_misses_host(fmt, d, f, tabs[l], E, recs[l], len(recs[l]), l, xs[l], T, ref, 2)
        np.testing.assert_array_equal(ys[l], ref)


def test_miss_engine_reports_bad_records_and_keeps_y():
    d, f, E, T = 512, 256, 3, 2
    canon = _experts(2, d, f, [0, 1])
    tab = native.expert_table(E, canon)
    x = synth.gen_x(1, 0, T, d)
    y = np.ones((T, d), np.float32)
    recs = np.array([(0, 1, 1, 0, 0.5), (0, 2, 0, 0, 0.5)], MISS_DT)   # expert 2 not given
    count = np.array([2], np.int32)
    eng = native.MissEngine(2)
    try:
        eng.submit(2, d, f, tab, E, recs, count, 2, 0, x, T, y)
        with pytest.raises(native.MoeError) as ei:
            eng.wait()
        assert ei.value.code == 1
        assert np.all(y == 1.0)
        # the engine stays usable
        good = np.array([(0, 1, 1, 0, 0.5)], MISS_DT)
        eng.submit(2, d, f, tab, E, good, np.array([1], np.int32), 1, 0, x, T, y)
        eng.wait()
        assert not np.all(y == 1.0)
    finally:
        eng.close()
