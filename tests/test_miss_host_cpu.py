"""Host completion of the miss list (moe_complete_misses_host) against the oracle.

The library computes the missed experts on the host from their packed records;
the oracle computes the same SwiGLU experts in fp64 from the canonical storage.
Every record adds gate * FFN_e(x_t) into y[t]; y is compared with
y0 + sum of the oracle's terms, within max|y - y_ref| / max|y_ref| <= 1e-5
(fp32 dot products of length <= 2048 against fp64).
"""
import numpy as np
import pytest

from bit_expert_ffn_fp32_b200 import native, synth

MISS_DT = np.dtype([("layer", "<i4"), ("expert", "<i4"), ("token", "<i4"), ("j", "<i4"), ("gate", "<f4")])
TOL = 1e-5


def _qm(m):
    return native.qmatrix(m["codes"], m["scale"], m["min"], m["hi"])


def _host_pool(fmt, d, f, experts, seed=11, layer=0):
    """Packed records of `experts` in a host buffer, slot s = position in `experts`."""
    nbytes = native.expert_bytes(fmt, d, f)
    stride = (nbytes + 255) // 256 * 256
    buf = np.zeros(stride * len(experts) + 256, np.uint8)
    base = (-buf.ctypes.data) % 256  # 256-byte aligned records
    canon = {}
    for s, e in enumerate(experts):
        ex = synth.gen_expert(seed, layer, e, fmt, d, f)
        canon[e] = ex
        native.pack_expert_host(fmt, d, f, _qm(ex["gate"]), _qm(ex["up"]), _qm(ex["down"]),
                                buf.ctypes.data + base + s * stride)
    pool = native.QPool(buf.ctypes.data + base, stride, len(experts), fmt, d, f)
    return pool, buf, canon


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
    experts = list(range(E))
    pool, buf, canon = _host_pool(fmt, d, f, experts)
    slot_of = np.arange(E, dtype=np.int32)
    x = synth.gen_x(3, 0, T, d, stream=7)
    # two misses on one token, two tokens on one expert, gates of either sign of size
    recs = np.array([(0, 4, 0, 2, 0.30), (0, 1, 3, 0, 0.05), (0, 4, 2, 7, 0.125), (0, 0, 0, 5, 0.2),
                     (0, 5, 4, 1, 0.9)], MISS_DT)
    y0 = np.random.default_rng(2).standard_normal((T, d)).astype(np.float32)
    y = y0.copy()
    native.complete_misses_host(pool, slot_of, E, recs, len(recs), 0, x, T, y, nthreads)
    ref = y0.astype(np.float64) + _oracle_terms(orc, canon, fmt, x, recs)
    err = np.max(np.abs(y - ref)) / np.max(np.abs(ref))
    assert err <= TOL, err
    untouched = [t for t in range(T) if t not in set(recs["token"].tolist())]
    np.testing.assert_array_equal(y[untouched], y0[untouched])


def test_complete_misses_full_size_expert_and_thread_independence(orc):
    """d=2048, f=768 (the decode shapes), Q2, one expert missed by two tokens;
    the result is the same bit for bit for 1 and 4 threads."""
    d, f, E, T = 2048, 768, 2, 3
    pool, buf, canon = _host_pool(2, d, f, [0, 1], seed=5)
    slot_of = np.array([1, 0], np.int32)  # expert 0 in slot 1, expert 1 in slot 0
    x = synth.gen_x(5, 0, T, d, stream=1)
    recs = np.array([(0, 0, 2, 3, 0.4), (0, 1, 0, 0, 0.6), (0, 0, 0, 9, 0.25)], MISS_DT)
    ys = []
    for nth in (1, 4):
        y = np.zeros((T, d), np.float32)
        native.complete_misses_host(pool, slot_of, E, recs, len(recs), 0, x, T, y, nth)
        ys.append(y)
    np.testing.assert_array_equal(ys[0], ys[1])
    # slot s holds generated expert s, so expert 0 (slot 1) has generated expert 1's weights
    ref = _oracle_terms(orc, {0: canon[1], 1: canon[0]}, 2, x, recs)
    err = np.max(np.abs(ys[0] - ref)) / np.max(np.abs(ref))
    assert err <= TOL, err
    assert np.all(ys[0][1] == 0)


def test_complete_misses_rejects_bad_records_before_writing():
    d, f, E, T = 512, 256, 3, 2
    pool, buf, _ = _host_pool(2, d, f, [0, 1])
    slot_of = np.array([0, 1, -1], np.int32)  # expert 2 has no host slot
    x = synth.gen_x(1, 0, T, d)
    y = np.ones((T, d), np.float32)
    L = native.lib
    import ctypes as C

    def call(recs, layer=0, E_=E, T_=T):
        return L.moe_complete_misses_host(C.byref(pool), slot_of.ctypes.data, E_, recs.ctypes.data, len(recs),
                                          layer, x.ctypes.data, T_, y.ctypes.data, 1)

    good = (0, 1, 1, 0, 0.5)
    for bad in [(1, 1, 1, 0, 0.5),    # another layer
                (0, 3, 1, 0, 0.5),    # expert outside [0, E)
                (0, -1, 1, 0, 0.5),
                (0, 1, 2, 0, 0.5),    # token outside [0, T)
                (0, 2, 0, 0, 0.5)]:   # expert without a host slot
        assert call(np.array([good, bad], MISS_DT)) == 1
        assert np.all(y == 1.0)
    assert call(np.zeros(0, MISS_DT)) == 0
    assert np.all(y == 1.0)
