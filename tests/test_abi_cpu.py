"""C-ABI checks that need no GPU: exports, host-side argument validation,
packed-record bijection, and the fragment-extraction rules of the kernels
replayed in Python on a host-packed record."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from conftest import ROOT
from bit_expert_ffn_fp32_b200 import configs, native, synth

HEADER = os.path.join(ROOT, "include", "moe.h")


def declared_functions():
    src = open(HEADER, encoding="utf-8").read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 14
    lib = C.CDLL(native.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(native.SIGNATURES), set(names) ^ set(native.SIGNATURES)


def test_status_strings_and_version():
    for code, name in native.STATUS_NAMES.items():
        assert native.lib.moe_status_str(code).decode().startswith(name)
    assert native.lib.moe_version() >= 100


@pytest.mark.parametrize("fmt,d,f,expect", [(2, 2048, 768, 1474560), (3, 2048, 768, 1916928), (2, 512, 256, 122880),
                                            (4, 2048, 768, 0), (2, 2000, 768, 0), (3, 2048, 100, 0)])
def test_expert_bytes(fmt, d, f, expect):
    assert native.expert_bytes(fmt, d, f) == expect
    if expect:
        assert expect == configs.expert_bytes(fmt, d, f) and expect % 256 == 0


def test_host_validation_rejects_before_launch():
    L = native.lib
    dummy = 0x1000  # never dereferenced: every call below must fail validation first
    # null required pointers
    assert L.moe_route(None, None, None, 4, 2048, 512, 10, None, None, None, None, None) == 1
    # d not a multiple of 128, k > 16, k > E
    assert L.moe_route(dummy, dummy, None, 4, 2000, 512, 10, dummy, dummy, dummy, None, None) == 2
    assert L.moe_route(dummy, dummy, None, 4, 2048, 512, 17, dummy, dummy, dummy, None, None) == 2
    assert L.moe_route(dummy, dummy, None, 4, 2048, 8, 10, dummy, dummy, dummy, None, None) == 2
    # overflow of T*E
    assert L.moe_route(dummy, dummy, None, 1 << 30, 2048, 512, 10, dummy, dummy, dummy, None, None) == 5
    # T == 0 is a no-op
    assert L.moe_route(None, None, None, 0, 2048, 512, 10, None, None, None, None, None) == 0
    # x or Wr not 16-byte aligned
    assert L.moe_route(dummy + 8, dummy, None, 4, 2048, 512, 10, dummy, dummy, dummy, None, None) == 1
    assert L.moe_route(dummy, dummy + 4, None, 4, 2048, 512, 10, dummy, dummy, dummy, None, None) == 1
    # permute: too small workspace for a multi-tile input
    need = native.permute_workspace_bytes(8192, 10, 512)
    assert need > 0
    assert L.moe_permute(dummy, 8192, 10, 512, dummy, dummy, dummy, dummy, dummy, dummy, dummy, need - 4,
                         None, None) == 3
    assert L.moe_permute(dummy, 8, 10, 5000, dummy, dummy, dummy, dummy, dummy, dummy, None, 0, None, None) == 2
    # cache lookup: null offsets
    assert L.moe_cache_lookup(dummy, 10, 0, dummy, dummy, None, dummy, dummy, 1, 10, 512, dummy, dummy, dummy, 10,
                              None, None, None) == 1
    # ffn: format mismatch, bad dims, small workspace
    pool = native.QPool(dummy * 256, 1474560, 10, 3, 2048, 768)
    args = [dummy, dummy, 1, 2048, 768, 512, 10, dummy, dummy, dummy, dummy, None, dummy, dummy, 1 << 20, None, None]
    assert L.moe_expert_ffn_q2(C.byref(pool), *args) == 1
    pool.fmt = 2
    assert L.moe_expert_ffn_q2(C.byref(pool), *args[:3], 2000, *args[4:]) == 1   # d != pool d
    small = list(args)
    small[14] = 16
    assert L.moe_expert_ffn_q2(C.byref(pool), *small) == 3
    pool.slot_bytes = 1000
    assert L.moe_expert_ffn_q2(C.byref(pool), *args) == 1
    # one-launch decode layer: d above the 2048 it stages, T above 8
    wide = native.QPool(dummy * 256, 1 << 23, 10, 2, 4096, 768)
    dec = [dummy, 0, 0, dummy, dummy, None, 1, 4096, 768, 512, 10] + [None] * 12 + [0, None, dummy, dummy, 1 << 24,
                                                                                  None, None]
    assert L.moe_layer_decode(C.byref(wide), *dec) == 2
    dec9 = list(dec)
    dec9[6], dec9[7], dec9[8] = 9, 2048, 768
    assert L.moe_layer_decode(C.byref(pool), *dec9) == 2
    # stacked layers: no shared-slot table, zero layers, misaligned x
    st = [C.byref(pool), 4, dummy, None, 0, dummy, dummy, None, 1, 2048, 768, 512, 10, None, None, None, None, None, 0,
          None, dummy, dummy, 1 << 24, None, None]
    assert L.moe_stack_decode(*st) == 1
    st0 = list(st)
    st0[1] = 0
    assert L.moe_stack_decode(*st0) == 1
    st3 = list(st)
    st3[3], st3[5] = dummy, dummy + 2
    assert L.moe_stack_decode(*st3) == 1
    # wait probe: null pointers
    assert L.moe_debug_wait_probe(None, 1, dummy, dummy, None) == 1
    assert L.moe_debug_wait_probe(dummy, 1, None, dummy, None) == 1
    # combine: d not a multiple of 4
    assert L.moe_combine(dummy, dummy, dummy, None, None, 2, 10, 2046, dummy, None) == 2
    # pack: missing hi plane for Q3
    q = native.QMatrix(dummy, None, dummy, None)
    assert L.moe_pack_expert(3, 2048, 768, C.byref(q), C.byref(q), C.byref(q), dummy * 256, None) == 1


def test_expert_ffn_workspace_per_path_and_noalloc_limit():
    """Below 512 pairs only the weight-streaming path runs (h as fp32); from 512
    pairs on the tensor-core layout (fp16 h + fp16 activation rows) is included.
    The allocation-free call's 4 MiB array therefore takes up to 744 pairs at
    d=2048, f=768, and 745 pairs are refused before any CUDA call."""
    d, f = 2048, 768
    assert native.expert_ffn_workspace_bytes(1, 10, d, f) == 10 * f * 4
    assert native.expert_ffn_workspace_bytes(51, 10, d, f) == 510 * f * 4
    assert native.expert_ffn_workspace_bytes(512, 1, d, f) == 512 * (2 * f + 2 * d)
    lim = 4 << 20
    assert native.expert_ffn_workspace_bytes(744, 1, d, f) <= lim < native.expert_ffn_workspace_bytes(745, 1, d, f)
    pool = native.QPool(0x1000 * 256, 1474560, 10, 2, d, f)
    dummy = 0x1000
    rc = native.lib.moe_expert_ffn_q2_noalloc(C.byref(pool), dummy, dummy, 745, d, f, 512, 1, dummy, dummy, dummy,
                                              dummy, None, dummy, None, None)
    assert rc == 3


def _canon(fmt, d, f, seed):
    return synth.gen_expert(seed, 0, 0, fmt, d, f)


def _qm(m):
    return native.qmatrix(m["codes"], m["scale"], m["min"], m["hi"])


@pytest.mark.parametrize("fmt", [2, 3])
def test_pack_unpack_roundtrip(fmt):
    d, f = 512, 256
    ex = _canon(fmt, d, f, 5)
    nbytes = native.expert_bytes(fmt, d, f)
    rec = np.zeros(nbytes, np.uint8)
    native.pack_expert_host(fmt, d, f, _qm(ex["gate"]), _qm(ex["up"]), _qm(ex["down"]), rec.ctypes.data)
    out = {m: {k: (None if v is None else np.zeros_like(v)) for k, v in ex[m].items()} for m in ex}
    native.unpack_expert_host(fmt, d, f, rec.ctypes.data, _qm(out["gate"]), _qm(out["up"]), _qm(out["down"]))
    for m in ex:
        for key, v in ex[m].items():
            if v is not None:
                np.testing.assert_array_equal(out[m][key], v, err_msg=f"{m}.{key}")
    # bijection on the record side too: random record -> canonical -> record
    rng = np.random.default_rng(1)
    rec2 = rng.integers(0, 256, nbytes, dtype=np.uint8)
    out2 = {m: {k: (None if v is None else np.zeros_like(v)) for k, v in ex[m].items()} for m in ex}
    native.unpack_expert_host(fmt, d, f, rec2.ctypes.data, _qm(out2["gate"]), _qm(out2["up"]), _qm(out2["down"]))
    rec3 = np.zeros(nbytes, np.uint8)
    native.pack_expert_host(fmt, d, f, _qm(out2["gate"]), _qm(out2["up"]), _qm(out2["down"]), rec3.ctypes.data)
    # every byte of the record is payload except the Q3 spare-free padding (none) -> identical
    np.testing.assert_array_equal(rec3, rec2)


# ---------------------------------------------------------------- kernel extraction rules replayed
def _slot_k(rho, t, h):
    return 16 * (rho >> 1) + 8 * (rho & 1) + 2 * t + h


def _q2_reg(w, rho):
    return (w & (0x00030003 << (2 * rho))) if rho < 5 else ((w >> 10) & (0x00030003 << (2 * (rho - 5))))


def _q2_exp(rho):
    return 2 * rho if rho < 5 else 2 * rho - 10


def _q3_reg(W, u, r):
    if u < 30:
        wp, kind = divmod(u, 5)
        if kind == 0:
            return ((W[2 * wp] >> 9) & 0x00070007) if r else (W[2 * wp] & 0x00070007)
        if kind == 1:
            return ((W[2 * wp] >> 9) & 0x00380038) if r else (W[2 * wp] & 0x00380038)
        if kind == 2:
            return ((W[2 * wp + 1] >> 9) & 0x00070007) if r else (W[2 * wp + 1] & 0x00070007)
        if kind == 3:
            return ((W[2 * wp + 1] >> 9) & 0x00380038) if r else (W[2 * wp + 1] & 0x00380038)
        return W[2 * wp + r] & 0x01C001C0
    b = 6 * (u - 30) + 3 * r
    return ((W[b] >> 15) & 0x00010001) | ((W[b + 1] >> 14) & 0x00020002) | ((W[b + 2] >> 13) & 0x00040004)


def _q3_exp(u):
    if u >= 30:
        return 0
    kind = u % 5
    return 6 if kind == 4 else (3 if kind in (1, 3) else 0)


def _canon_code(m, fmt, row, k):
    q = (int(m["codes"][row, k // 4]) >> (2 * (k % 4))) & 3
    if fmt == 3:
        q |= ((int(m["hi"][row, k // 8]) >> (k % 8)) & 1) << 2
    return q


@pytest.mark.parametrize("fmt", [2, 3])
def test_fragment_extraction_matches_canonical(fmt):
    """Replays the kernels' register extraction on a host-packed record: the fp16
    half of fragment register (rho, row, half) must be the subnormal q * 2^exp
    of the canonical code at (row, k)."""
    d, f = 256, 256
    ex = _canon(fmt, d, f, 9)
    nbytes = native.expert_bytes(fmt, d, f)
    rec = np.zeros(nbytes, np.uint8)
    native.pack_expert_host(fmt, d, f, _qm(ex["gate"]), _qm(ex["up"]), _qm(ex["down"]), rec.ctypes.data)
    words = rec.view("<u4")
    m = ex["gate"]          # gate matrix occupies the record's first region: codes first
    K = d
    NB = K // 64
    for rg in (0, 5, 15):
        for L in range(32):
            g, t = L >> 2, L & 3
            if fmt == 2:
                for p in range(NB // 2):
                    base = ((rg * (NB // 2) + p) * 32 + L) * 16 // 4
                    w4 = [int(words[base + i]) for i in range(4)]
                    for bb in range(2):
                        for r in range(2):
                            w = w4[2 * bb + r]
                            for rho in range(8):
                                reg = _q2_reg(w, rho)
                                for h in range(2):
                                    half = (reg >> (16 * h)) & 0xFFFF
                                    k = 64 * (2 * p + bb) + _slot_k(rho, t, h)
                                    q = _canon_code(m, 2, 16 * rg + g + 8 * r, k)
                                    assert half == q << _q2_exp(rho), (rg, L, p, bb, r, rho, h)
            else:
                for qd in range(NB // 4):
                    W = []
                    for wi in range(12):
                        off = (rg * (NB // 4) + qd) * 1536 + (wi >> 2) * 512 + L * 16 + (wi & 3) * 4
                        W.append(int(words[off // 4]))
                    for u in range(32):
                        for r in range(2):
                            reg = _q3_reg(W, u, r)
                            for h in range(2):
                                half = (reg >> (16 * h)) & 0xFFFF
                                k = 256 * qd + 64 * (u >> 3) + _slot_k(u & 7, t, h)
                                q = _canon_code(m, 3, 16 * rg + g + 8 * r, k)
                                assert half == q << _q3_exp(u), (rg, L, qd, u, r, h)
