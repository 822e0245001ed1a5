"""ctypes binding of libmoe (include/moe.h): argument marshalling only.

Every function here passes raw device pointers, sizes and the current CUDA
stream to the C ABI of the same name; all the layer's work runs in the
library's kernels. Tensors are torch tensors on the GPU (PyTorch provides the
device memory and the stream), except where a name ends in ``_host``.

Importing this module raises if libmoe.so has not been built: there is no
fallback path.
"""
from __future__ import annotations

import ctypes as C
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoe.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
                4: "MOE_ERR_CUDA", 5: "MOE_ERR_OVERFLOW", 6: "MOE_ERR_HOST"}
DEV_BAD_INDEX, DEV_BAD_SLOT, DEV_NONFINITE, DEV_MISS_OVERFLOW, DEV_TIMEOUT = 0x1, 0x2, 0x4, 0x8, 0x10

_P = C.c_void_p
_I = C.c_int
_I32 = C.c_int32
_SZ = C.c_size_t


class QPool(C.Structure):
    _fields_ = [("base", _P), ("slot_bytes", C.c_int64), ("num_slots", _I32), ("fmt", _I32), ("d", _I32),
                ("f", _I32)]


class QMatrix(C.Structure):
    _fields_ = [("codes", _P), ("hi", _P), ("scale", _P), ("min", _P)]


class Swap(C.Structure):
    _fields_ = [("slot", _I32), ("layer_in", _I32), ("expert_in", _I32), ("layer_out", _I32), ("expert_out", _I32)]


class Miss(C.Structure):
    _fields_ = [("layer", _I32), ("expert", _I32), ("token", _I32), ("j", _I32), ("gate", C.c_float)]


MISS_BYTES = C.sizeof(Miss)

# name -> (restype, argtypes), mirroring include/moe.h
SIGNATURES = {
    "moe_status_str": (C.c_char_p, [_I]),
    "moe_version": (_I, []),
    "moe_expert_bytes": (_SZ, [_I, _I, _I]),
    "moe_pack_expert": (_I, [_I, _I, _I, C.POINTER(QMatrix), C.POINTER(QMatrix), C.POINTER(QMatrix), _P, _P]),
    "moe_pack_expert_host": (_I, [_I, _I, _I, C.POINTER(QMatrix), C.POINTER(QMatrix), C.POINTER(QMatrix), _P]),
    "moe_unpack_expert_host": (_I, [_I, _I, _I, _P, C.POINTER(QMatrix), C.POINTER(QMatrix), C.POINTER(QMatrix)]),
    "moe_route": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P]),
    "moe_permute_workspace_bytes": (_SZ, [_I, _I, _I]),
    "moe_permute": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _SZ, _P, _P]),
    "moe_cache_lookup": (_I, [_P, _I32, _I32, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _I32, _P, _P, _P]),
    "moe_expert_ffn_workspace_bytes": (_SZ, [_I, _I, _I, _I]),
    "moe_expert_ffn_q2": (_I, [C.POINTER(QPool), _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _SZ, _P,
                               _P]),
    "moe_expert_ffn_q3": (_I, [C.POINTER(QPool), _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _SZ, _P,
                               _P]),
    "moe_expert_ffn_q2_noalloc": (_I, [C.POINTER(QPool), _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P,
                                       _P]),
    "moe_combine": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P, _P]),
    "moe_layer_decode_workspace_bytes": (_SZ, [_I, _I, _I, _I]),
    "moe_layer_decode": (_I, [C.POINTER(QPool), _P, _I32, _I32, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P,
                              _P, _P, _P, _P, _P, _P, _P, _I32, _P, _P, _P, _SZ, _P, _P]),
    "moe_stack_decode_workspace_bytes": (_SZ, [_I, _I, _I, _I]),
    "moe_stack_decode": (_I, [C.POINTER(QPool), _I, _P, _P, _I32, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P,
                              _P, _I32, _P, _P, _P, _SZ, _P, _P]),
    "moe_complete_misses_host": (_I, [_I, _I, _I, _P, _I, _P, _I32, _I32, _P, _I, _P, _I]),
    "moe_debug_wait_probe": (_I, [_P, C.c_uint32, _P, _P, _P]),
    "moe_miss_engine_create": (_I, [_I, C.POINTER(_P)]),
    "moe_miss_engine_submit": (_I, [_P, _I, _I, _I, _P, _I, _P, _P, _I32, _I32, _P, _I, _P]),
    "moe_miss_engine_wait": (_I, [_P]),
    "moe_miss_engine_destroy": (None, [_P]),
    "moe_cache_policy_bytes": (_SZ, [_I, _I]),
    "moe_cache_policy_init": (_I, [_P, _SZ, _I, _I, _I, _I, _I]),
    "moe_cache_policy_observe": (_I, [_P, _I, _P, _I, _I]),
    "moe_cache_policy_observe_counts": (_I, [_P, _P, _I]),
    "moe_cache_policy_plan": (_I32, [_P, _P, _P, _I32]),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libmoe.so is not built ({LIB_PATH}); run `python -m bit_expert_ffn_fp32_b200.build`")
    lib = C.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn}: {lib.moe_status_str(code).decode()}")
        self.code = code


def check(fn: str, code: int) -> None:
    if code != MOE_OK:
        raise MoeError(fn, code)


def ptr(t) -> int | None:
    """Device (or host) address of a tensor/array, None for None."""
    if t is None:
        return None
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    return t.ctypes.data  # numpy


def stream_handle(stream=None) -> int | None:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream or None


def qmatrix(codes, scale, mn=None, hi=None) -> QMatrix:
    return QMatrix(ptr(codes), ptr(hi), ptr(scale), ptr(mn))


def qpool(base, slot_bytes: int, num_slots: int, fmt: int, d: int, f: int) -> QPool:
    return QPool(ptr(base), slot_bytes, num_slots, fmt, d, f)


# ------------------------------------------------------------------ thin wrappers
def expert_bytes(fmt: int, d: int, f: int) -> int:
    return int(lib.moe_expert_bytes(fmt, d, f))


def pack_expert(fmt, d, f, gate: QMatrix, up: QMatrix, down: QMatrix, dst_ptr: int, stream=None) -> None:
    check("moe_pack_expert", lib.moe_pack_expert(fmt, d, f, C.byref(gate), C.byref(up), C.byref(down), dst_ptr,
                                                 stream_handle(stream)))


def pack_expert_host(fmt, d, f, gate: QMatrix, up: QMatrix, down: QMatrix, dst_ptr: int) -> None:
    check("moe_pack_expert_host", lib.moe_pack_expert_host(fmt, d, f, C.byref(gate), C.byref(up), C.byref(down),
                                                           dst_ptr))


def unpack_expert_host(fmt, d, f, src_ptr: int, gate: QMatrix, up: QMatrix, down: QMatrix) -> None:
    check("moe_unpack_expert_host", lib.moe_unpack_expert_host(fmt, d, f, src_ptr, C.byref(gate), C.byref(up),
                                                               C.byref(down)))


def route(x, Wr, bias, T, d, E, k, logits, topk_idx, topk_w, dev_status=None, stream=None) -> None:
    check("moe_route", lib.moe_route(ptr(x), ptr(Wr), ptr(bias), T, d, E, k, ptr(logits), ptr(topk_idx),
                                     ptr(topk_w), ptr(dev_status), stream_handle(stream)))


def permute_workspace_bytes(T, k, E) -> int:
    return int(lib.moe_permute_workspace_bytes(T, k, E))


def permute(topk_idx, T, k, E, counts, offsets, sorted_tok, sorted_j, inv, active, ws=None, ws_bytes=0,
            dev_status=None, stream=None) -> None:
    check("moe_permute", lib.moe_permute(ptr(topk_idx), T, k, E, ptr(counts), ptr(offsets), ptr(sorted_tok),
                                         ptr(sorted_j), ptr(inv), ptr(active), ptr(ws), ws_bytes, ptr(dev_status),
                                         stream_handle(stream)))


def cache_lookup(slot_of, num_slots, layer, topk_idx, topk_w, offsets, sorted_tok, sorted_j, T, k, E,
                 slot_of_pair, miss, miss_count, miss_cap, dev_status=None, stream=None, expert_counts=None) -> None:
    check("moe_cache_lookup", lib.moe_cache_lookup(ptr(slot_of), num_slots, layer, ptr(topk_idx), ptr(topk_w),
                                                   ptr(offsets), ptr(sorted_tok), ptr(sorted_j), T, k, E,
                                                   ptr(slot_of_pair), ptr(miss), ptr(miss_count), miss_cap,
                                                   ptr(expert_counts), ptr(dev_status), stream_handle(stream)))


def expert_ffn_workspace_bytes(T, k, d, f) -> int:
    return int(lib.moe_expert_ffn_workspace_bytes(T, k, d, f))


def expert_ffn(pool: QPool, slot_of, x, T, d, f, E, k, offsets, sorted_tok, sorted_j, active, topk_w, out, ws,
               ws_bytes, dev_status=None, stream=None) -> None:
    fn = lib.moe_expert_ffn_q2 if pool.fmt == 2 else lib.moe_expert_ffn_q3
    name = "moe_expert_ffn_q2" if pool.fmt == 2 else "moe_expert_ffn_q3"
    check(name, fn(C.byref(pool), ptr(slot_of), ptr(x), T, d, f, E, k, ptr(offsets), ptr(sorted_tok),
                   ptr(sorted_j), ptr(active), ptr(topk_w), ptr(out), ptr(ws), ws_bytes, ptr(dev_status),
                   stream_handle(stream)))


def expert_ffn_q2_noalloc(pool: QPool, slot_of, x, T, d, f, E, k, offsets, sorted_tok, sorted_j, active, topk_w,
                          out, dev_status=None, stream=None) -> None:
    """moe_expert_ffn_q2 with the library's built-in scratch instead of a workspace."""
    check("moe_expert_ffn_q2_noalloc",
          lib.moe_expert_ffn_q2_noalloc(C.byref(pool), ptr(slot_of), ptr(x), T, d, f, E, k, ptr(offsets),
                                        ptr(sorted_tok), ptr(sorted_j), ptr(active), ptr(topk_w), ptr(out),
                                        ptr(dev_status), stream_handle(stream)))


def combine(y_perm, inv, topk_w, slot_of_pair, y_shared, T, k, d, y, stream=None) -> None:
    check("moe_combine", lib.moe_combine(ptr(y_perm), ptr(inv), ptr(topk_w), ptr(slot_of_pair), ptr(y_shared), T,
                                         k, d, ptr(y), stream_handle(stream)))


def layer_decode_workspace_bytes(T, k, f, E) -> int:
    return int(lib.moe_layer_decode_workspace_bytes(T, k, f, E))


def layer_decode(pool: QPool, slot_of, shared_slot: int, layer: int, x, Wr, bias, T, d, f, E, k, logits=None,
                 topk_idx=None, topk_w=None, counts=None, offsets=None, sorted_tok=None, sorted_j=None, inv=None,
                 active=None, slot_of_pair=None, miss=None, miss_count=None, miss_cap=0, y=None, ws=None,
                 ws_bytes=0, dev_status=None, stream=None, expert_counts=None) -> None:
    check("moe_layer_decode",
          lib.moe_layer_decode(C.byref(pool), ptr(slot_of), shared_slot, layer, ptr(x), ptr(Wr), ptr(bias), T, d, f,
                               E, k, ptr(logits), ptr(topk_idx), ptr(topk_w), ptr(counts), ptr(offsets),
                               ptr(sorted_tok), ptr(sorted_j), ptr(inv), ptr(active), ptr(slot_of_pair), ptr(miss),
                               ptr(miss_count), miss_cap, ptr(expert_counts), ptr(y), ptr(ws), ws_bytes,
                               ptr(dev_status), stream_handle(stream)))


def stack_decode(pool: QPool, L: int, slot_of, shared_slot, layer0: int, x, Wr, bias, T, d, f, E, k, topk_idx=None,
                 topk_w=None, slot_of_pair=None, miss=None, miss_count=None, miss_cap=0, y=None, ws=None,
                 ws_bytes=0, dev_status=None, stream=None, expert_counts=None) -> None:
    check("moe_stack_decode",
          lib.moe_stack_decode(C.byref(pool), L, ptr(slot_of), ptr(shared_slot), layer0, ptr(x), ptr(Wr), ptr(bias),
                               T, d, f, E, k, ptr(topk_idx), ptr(topk_w), ptr(slot_of_pair), ptr(miss),
                               ptr(miss_count), miss_cap, ptr(expert_counts), ptr(y), ptr(ws), ws_bytes,
                               ptr(dev_status), stream_handle(stream)))


def expert_table(E: int, experts: dict) -> C.Array:
    """moe_qmatrix [E][3] (gate, up, down) for the experts given as
    {e: canonical expert dict}; absent experts get NULL matrices. The arrays
    must stay alive while the table is used."""
    tab = (QMatrix * (3 * E))()
    for e, ex in experts.items():
        for i, m in enumerate(("gate", "up", "down")):
            tab[3 * e + i] = qmatrix(ex[m]["codes"], ex[m]["scale"], ex[m]["min"], ex[m]["hi"])
    return tab


def complete_misses_host(fmt: int, d: int, f: int, experts: C.Array, E: int, miss, n: int, layer: int, x, T: int, y,
                         nthreads: int = 0) -> None:
    """Host completion of a layer's miss list (host arrays: experts from
    expert_table, miss records, x uint16 [T][d], y float32 [T][d] accumulated
    in place)."""
    check("moe_complete_misses_host",
          lib.moe_complete_misses_host(fmt, d, f, C.cast(experts, _P), E, ptr(miss), n, layer, ptr(x), T, ptr(y),
                                       nthreads))


class MissEngine:
    """moe_miss_engine: host worker threads completing miss lists as they are
    published (see include/moe.h). Submitted arrays must stay alive until
    wait() returns; the engine keeps references to them until then."""

    def __init__(self, nthreads: int = 0):
        h = _P()
        check("moe_miss_engine_create", lib.moe_miss_engine_create(nthreads, C.byref(h)))
        self.h = h
        self._keep = []

    def submit(self, fmt: int, d: int, f: int, experts: C.Array, E: int, miss, count, miss_cap: int, layer: int, x,
               T: int, y) -> None:
        """miss: host records (e.g. a pinned tensor the GPU writes), count: host
        int32 whose value becomes >= 0 when the records are complete."""
        self._keep.append((experts, miss, count, x, y))
        check("moe_miss_engine_submit",
              lib.moe_miss_engine_submit(self.h, fmt, d, f, C.cast(experts, _P), E, ptr(miss), ptr(count), miss_cap,
                                         layer, ptr(x), T, ptr(y)))

    def wait(self) -> None:
        code = lib.moe_miss_engine_wait(self.h)
        self._keep.clear()
        check("moe_miss_engine_wait", code)

    def close(self) -> None:
        if self.h:
            lib.moe_miss_engine_destroy(self.h)
            self.h = None
            self._keep.clear()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class CachePolicy:
    """Host expert-cache policy (moe_cache_policy_*): counts of routed pairs,
    halved every `epoch` tokens, and slot plans against an [L][E] slot table."""

    def __init__(self, L: int, E: int, S: int, epoch: int, margin: int = 0):
        import numpy as np

        n = int(lib.moe_cache_policy_bytes(L, E))
        if n == 0:
            raise MoeError("moe_cache_policy_bytes", 2)
        self.L, self.E, self.S = L, E, S
        self.state = np.zeros(n, np.uint8)
        check("moe_cache_policy_init", lib.moe_cache_policy_init(self.state.ctypes.data, n, L, E, S, epoch, margin))

    def observe(self, layer: int, topk_idx) -> None:
        import numpy as np

        idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
        T, k = idx.shape
        check("moe_cache_policy_observe", lib.moe_cache_policy_observe(self.state.ctypes.data, layer, idx.ctypes.data,
                                                                       T, k))

    def observe_counts(self, counts, tokens: int) -> None:
        """A window of `tokens` token steps from per-expert counts (int32 [L][E])."""
        import numpy as np

        c = np.ascontiguousarray(counts, dtype=np.int32)
        check("moe_cache_policy_observe_counts",
              lib.moe_cache_policy_observe_counts(self.state.ctypes.data, c.ctypes.data, tokens))

    def plan(self, slot_of, max_swaps: int) -> list:
        """Update slot_of (int32 [L][E] numpy, in place); the changes as tuples
        (slot, layer_in, expert_in, layer_out, expert_out)."""
        buf = (Swap * max(1, max_swaps))()
        n = int(lib.moe_cache_policy_plan(self.state.ctypes.data, slot_of.ctypes.data, buf, max_swaps))
        if n < 0:
            raise MoeError("moe_cache_policy_plan", -n)
        return [(buf[i].slot, buf[i].layer_in, buf[i].expert_in, buf[i].layer_out, buf[i].expert_out)
                for i in range(n)]


def debug_wait_probe(counter, target: int, elapsed_ns, dev_status, stream=None) -> None:
    """moe_debug_wait_probe: the library's bounded waits against a counter below
    target and an mbarrier phase nothing completes (device tensors)."""
    check("moe_debug_wait_probe", lib.moe_debug_wait_probe(ptr(counter), target, ptr(elapsed_ns), ptr(dev_status),
                                                           stream_handle(stream)))
