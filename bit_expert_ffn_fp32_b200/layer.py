"""Device-resident MoE layers driven through the C ABI.

A ``MoEStack`` owns, for one or more layers of a workload, the fp32 router
weights (+ optional Zipf bias), the per-layer expert->slot table, and one pool
of packed experts in HBM (resident routed experts plus one shared expert per
layer). ``forward`` enqueues the layer's steps on the current stream:

    moe_route -> moe_permute -> moe_cache_lookup -> moe_expert_ffn (routed)
    -> moe_expert_ffn (shared, as E=1, k=1) -> moe_combine

Inputs are the seeded synthetic tensors of ``synth``; weights are generated on
the host and packed on the device by ``moe_pack_expert``.

A workload with ``q3_top > 0`` holds a mixed pool: per layer the ``q3_top``
most popular experts are stored Q3 and the rest (and the shared expert) in the
workload's format. Every slot is sized for the larger record; two pool
descriptions (one per format) share the base, and per-format slot tables keep
each ``moe_expert_ffn_q2/q3`` call to its own experts (the other format's
experts read as -1 there, so their rows are left to the other call).
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np
import torch

from . import native, synth
from .configs import ZIPF_ALPHA, Workload


def _t(a, device):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(device)


def upload_expert(ex: dict, fmt: int, d: int, f: int, dst_ptr: int, device, stream=None, sync: bool = True) -> None:
    """Pack one canonical expert (numpy) into the device record at dst_ptr.

    The canonical arrays are copied to temporary device tensors and packed on
    the current stream (or ``stream``). With sync=False nothing waits: the
    temporaries are released to torch's stream-ordered allocator, so later work
    on the same stream cannot reuse them before the pack kernel has run."""
    keep = []
    mats = []
    for m in ("gate", "up", "down"):
        c = ex[m]
        parts = [_t(c["codes"], device), _t(c["scale"].view(np.int16), device),
                 _t(None if c["min"] is None else c["min"].view(np.int16), device), _t(c["hi"], device)]
        keep.append(parts)
        mats.append(native.qmatrix(parts[0], parts[1], parts[2], parts[3]))
    if stream is not None and sync is False:
        raise ValueError("sync=False packs on the current stream only")
    native.pack_expert(fmt, d, f, mats[0], mats[1], mats[2], dst_ptr, stream)
    if sync:
        torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()
    del keep


@dataclass
class Buffers:
    T: int
    logits: torch.Tensor
    idx: torch.Tensor
    w: torch.Tensor
    counts: torch.Tensor
    offsets: torch.Tensor
    sorted_tok: torch.Tensor
    sorted_j: torch.Tensor
    inv: torch.Tensor
    active: torch.Tensor
    perm_ws: torch.Tensor | None
    sop: torch.Tensor
    miss: torch.Tensor
    miss_count: torch.Tensor
    h_ws: torch.Tensor
    h_sh: torch.Tensor
    y_perm: torch.Tensor
    y_sh: torch.Tensor
    y: torch.Tensor
    status: torch.Tensor
    sh_offsets: torch.Tensor
    sh_sorted_tok: torch.Tensor
    sh_sorted_j: torch.Tensor
    sh_active: torch.Tensor


MISS_DTYPE = np.dtype([("layer", "<i4"), ("expert", "<i4"), ("token", "<i4"), ("j", "<i4"), ("gate", "<f4")])


class MappedHostBuffer:
    """Pinned host memory mapped into the device address space: kernels write it
    through `data_ptr()` (a device address), the host reads `host` (a numpy
    view of the same bytes)."""

    def __init__(self, nbytes: int):
        from cuda.bindings import runtime as rt

        self._rt = rt
        err, hp = rt.cudaHostAlloc(max(int(nbytes), 16), rt.cudaHostAllocMapped | rt.cudaHostAllocPortable)
        if err != rt.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaHostAlloc failed: {err}")
        err, dp = rt.cudaHostGetDevicePointer(hp, 0)
        if err != rt.cudaError_t.cudaSuccess:
            rt.cudaFreeHost(hp)
            raise RuntimeError(f"cudaHostGetDevicePointer failed: {err}")
        self._hp, self._dp, self.nbytes = int(hp), int(dp), int(nbytes)
        import ctypes as _C
        self.host = np.ctypeslib.as_array((_C.c_uint8 * self.nbytes).from_address(self._hp))

    def data_ptr(self) -> int:
        return self._dp

    def view(self, dtype, shape=None) -> np.ndarray:
        v = self.host.view(dtype)
        return v if shape is None else v.reshape(shape)

    def __del__(self):
        try:
            self._rt.cudaFreeHost(self._hp)
        except Exception:
            pass


@dataclass
class StackBuffers:
    T: int
    idx: torch.Tensor        # [L][T*k]
    w: torch.Tensor          # [L][T*k]
    sop: torch.Tensor        # [L][T*k]
    miss: torch.Tensor       # [L][T*k] miss records (20 bytes each)
    miss_count: torch.Tensor  # [L]
    y: torch.Tensor          # [L][T][d]
    status: torch.Tensor


class MoEStack:
    def __init__(self, wl: Workload, device="cuda", seed: int | None = None, layers: int | None = None,
                 alpha: float = ZIPF_ALPHA):
        self.wl = wl
        self.device = torch.device(device)
        self.seed = wl.seed if seed is None else seed
        self.L = wl.layers if layers is None else layers
        self.R = wl.resident_count
        self.mixed = wl.q3_top > 0 and wl.fmt != 3
        self.fmts = (wl.fmt, 3) if self.mixed else (wl.fmt,)
        self.slot_bytes = max(native.expert_bytes(fm, wl.d, wl.f) for fm in self.fmts)
        if self.slot_bytes == 0:
            raise ValueError("unsupported shape")
        self.num_slots = self.L * self.R + self.L
        self.pool = torch.empty(self.num_slots * self.slot_bytes, dtype=torch.uint8, device=self.device)
        self.qpools = {fm: native.qpool(self.pool, self.slot_bytes, self.num_slots, fm, wl.d, wl.f)
                       for fm in self.fmts}
        self.qpool = self.qpools[wl.fmt]
        # per-layer router weights, biases and slot tables live in [L][...] device
        # tensors (the stacked call reads them with a layer stride); the lists
        # hold per-layer views
        self.Wr_all = torch.empty((self.L, wl.E, wl.d), dtype=torch.float32, device=self.device)
        self.bias_all = torch.empty((self.L, wl.E), dtype=torch.float32, device=self.device) if wl.zipf else None
        self.slot_of_all = torch.empty((self.L, wl.E), dtype=torch.int32, device=self.device)
        self.shared_slot_all = torch.arange(self.L * self.R, self.L * self.R + self.L, dtype=torch.int32,
                                            device=self.device)
        self.Wr, self.bias, self.rank, self.slot_of_host, self.slot_of, self.shared_slot = [], [], [], [], [], []
        # storage format of every routed expert, per layer (host); per-format
        # device slot tables [L][E] for the two calls of a mixed pool
        self.fmt_of_host = []
        self.slot_of_fmt_all = {fm: torch.empty((self.L, wl.E), dtype=torch.int32, device=self.device)
                                for fm in self.fmts} if self.mixed else {}
        for l in range(self.L):
            Wr = synth.gen_router(self.seed, l, wl.E, wl.d)
            rank = synth.gen_rank_perm(self.seed, l, wl.E)
            self.fmt_of_host.append(np.array([wl.expert_fmt(int(r)) for r in rank], np.int32))
            bias = synth.zipf_bias(rank, alpha) if wl.zipf else None
            if self.R >= wl.E:
                slot = np.arange(wl.E, dtype=np.int32) + l * self.R
            else:
                slot = synth.slot_table_by_rank(rank, self.R, l * self.R)
            self.Wr_all[l].copy_(torch.from_numpy(Wr))
            self.Wr.append(self.Wr_all[l])
            if bias is not None:
                self.bias_all[l].copy_(torch.from_numpy(bias))
            self.bias.append(None if bias is None else self.bias_all[l])
            self.rank.append(rank)
            self.slot_of_host.append(slot)
            self.slot_of_all[l].copy_(torch.from_numpy(slot))
            self.slot_of.append(self.slot_of_all[l])
            self.shared_slot.append(self.shared_slot_all[l:l + 1])
            self._copy_fmt_rows(l, non_blocking=False)
        # every resident expert and each layer's shared expert: generated on host
        # threads, packed on the current stream in order, one wait at the end
        jobs = [(l, e, int(self.slot_of_host[l][e])) for l in range(self.L) for e in range(wl.E)
                if self.slot_of_host[l][e] >= 0]
        jobs += [(l, wl.E, self.L * self.R + l) for l in range(self.L)]
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            for c0 in range(0, len(jobs), 64):  # at most 64 generated experts held at once
                chunk = jobs[c0:c0 + 64]
                for (l, e, slot), canon in zip(chunk, ex.map(lambda j: self.canonical_expert(j[0], j[1]), chunk)):
                    upload_expert(canon, self.expert_fmt(l, e), wl.d, wl.f,
                                  self.pool.data_ptr() + slot * self.slot_bytes, self.device, sync=False)
        torch.cuda.current_stream().synchronize()
        self._bufs: dict[int, Buffers] = {}
        # routed pairs per (layer, expert), added to by every forward (device
        # counters the cache policy reads in bulk); zero it to start a window
        self.count_experts = True
        self.expert_counts = torch.zeros((self.L, wl.E), dtype=torch.int32, device=self.device)
        self._ws: dict = {}

    # expert e == E is the layer's shared expert
    def expert_fmt(self, layer: int, e: int) -> int:
        return self.wl.fmt if e >= self.wl.E else int(self.fmt_of_host[layer][e])

    def canonical_expert(self, layer: int, e: int) -> dict:
        return synth.gen_expert(self.seed, layer, e, self.expert_fmt(layer, e), self.wl.d, self.wl.f)

    def _copy_fmt_rows(self, l: int, non_blocking: bool = True) -> None:
        """Per-format device slot tables of layer l from the host tables."""
        for fm, tab in self.slot_of_fmt_all.items():
            row = np.where(self.fmt_of_host[l] == fm, self.slot_of_host[l], -1).astype(np.int32)
            tab[l].copy_(torch.from_numpy(row), non_blocking=non_blocking)

    def apply_swaps(self, swaps) -> None:
        """Carry out a cache-policy plan: every (slot, layer_in, expert_in,
        layer_out, expert_out) packs expert_in's record into slot (on the
        current stream, after the work already queued there) and updates the
        slot tables, host and device."""
        changed = set()
        for slot, l_in, e_in, l_out, e_out in swaps:
            if not 0 <= slot < self.L * self.R:
                raise ValueError("slot %d outside the routed slots" % slot)
            if l_out >= 0:
                self.slot_of_host[l_out][e_out] = -1
                changed.add(l_out)
            self.slot_of_host[l_in][e_in] = slot
            changed.add(l_in)
            self._pack(l_in, e_in, slot)
        for l in changed:
            self.slot_of[l].copy_(torch.from_numpy(np.ascontiguousarray(self.slot_of_host[l], dtype=np.int32)))
            self._copy_fmt_rows(l, non_blocking=False)

    def _set_rows(self, layers) -> None:
        for l in sorted(layers):
            self.slot_of[l].copy_(torch.from_numpy(np.ascontiguousarray(self.slot_of_host[l], dtype=np.int32)),
                                  non_blocking=True)
            self._copy_fmt_rows(l)

    def prepare_swaps(self, swaps) -> list:
        """Pack every admitted expert of a plan into a pinned host record (host
        work, no GPU): [(slot, layer_in, expert_in, layer_out, expert_out, record)]."""
        out = []
        for slot, l_in, e_in, l_out, e_out in swaps:
            if not 0 <= slot < self.L * self.R:
                raise ValueError("slot %d outside the routed slots" % slot)
            ex = self.canonical_expert(l_in, e_in)
            rec = torch.empty(self.slot_bytes, dtype=torch.uint8).pin_memory()
            mats = [native.qmatrix(ex[m]["codes"], ex[m]["scale"], ex[m]["min"], ex[m]["hi"]) for m in
                    ("gate", "up", "down")]
            native.pack_expert_host(self.expert_fmt(l_in, e_in), self.wl.d, self.wl.f, *mats, rec.data_ptr())
            out.append((slot, l_in, e_in, l_out, e_out, rec))
        return out

    def begin_swaps(self, prepared: list, side_stream) -> dict:
        """Start a plan without stopping the layers: on the current stream the
        outgoing experts leave the slot tables (later layers count them as
        misses); once every layer queued before that point is done, the side
        stream copies the new records into their slots while the current stream
        goes on. commit_swaps() then makes the incoming experts resident."""
        main = torch.cuda.current_stream()
        changed = set()
        for slot, l_in, e_in, l_out, e_out, _ in prepared:
            if l_out >= 0:
                self.slot_of_host[l_out][e_out] = -1
                changed.add(l_out)
        self._set_rows(changed)
        unmapped = torch.cuda.Event()
        unmapped.record(main)
        side_stream.wait_event(unmapped)
        with torch.cuda.stream(side_stream):
            for slot, _, _, _, _, rec in prepared:
                dst = self.pool[slot * self.slot_bytes: slot * self.slot_bytes + rec.numel()]
                dst.copy_(rec, non_blocking=True)
        copied = torch.cuda.Event()
        copied.record(side_stream)
        return {"prepared": prepared, "copied": copied}

    def commit_swaps(self, handle: dict) -> None:
        """The current stream waits for the record copies, then the incoming
        experts take their slots in the slot tables."""
        torch.cuda.current_stream().wait_event(handle["copied"])
        changed = set()
        for slot, l_in, e_in, _, _, _ in handle["prepared"]:
            self.slot_of_host[l_in][e_in] = slot
            changed.add(l_in)
        self._set_rows(changed)

    def _pack(self, layer: int, e: int, slot: int) -> None:
        upload_expert(self.canonical_expert(layer, e), self.expert_fmt(layer, e), self.wl.d, self.wl.f,
                      self.pool.data_ptr() + slot * self.slot_bytes, self.device)

    def buffers(self, T: int, fresh: bool = False) -> Buffers:
        """Outputs and workspaces for T tokens: one cached set per T, or a new
        set with fresh=True (e.g. one per layer when several layers' outputs
        must stay readable)."""
        if T in self._bufs and not fresh:
            return self._bufs[T]
        wl, dev = self.wl, self.device
        n = T * wl.k
        i32 = dict(dtype=torch.int32, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        pws = native.permute_workspace_bytes(T, wl.k, wl.E)
        b = Buffers(
            T=T,
            logits=torch.empty(max(T, 1), wl.E, **f32), idx=torch.empty(max(n, 1), **i32),
            w=torch.empty(max(n, 1), **f32), counts=torch.empty(wl.E, **i32), offsets=torch.empty(wl.E + 1, **i32),
            sorted_tok=torch.empty(max(n, 1), **i32), sorted_j=torch.empty(max(n, 1), **i32),
            inv=torch.empty(max(n, 1), **i32), active=torch.empty(wl.E + 1, **i32),
            perm_ws=torch.empty(pws, dtype=torch.uint8, device=dev) if pws else None,
            sop=torch.empty(max(n, 1), **i32), miss=torch.empty(max(n, 1) * native.MISS_BYTES, dtype=torch.uint8,
                                                                device=dev),
            miss_count=torch.zeros(1, **i32),
            h_ws=torch.empty(max(native.expert_ffn_workspace_bytes(T, wl.k, wl.d, wl.f), 4), dtype=torch.uint8, device=dev),
            h_sh=torch.empty(max(native.expert_ffn_workspace_bytes(T, 1, wl.d, wl.f), 4), dtype=torch.uint8, device=dev),
            y_perm=torch.zeros(max(n, 1), wl.d, **f32), y_sh=torch.empty(max(T, 1), wl.d, **f32),
            y=torch.empty(max(T, 1), wl.d, **f32), status=torch.zeros(1, **i32),
            sh_offsets=torch.tensor([0, T], **i32), sh_sorted_tok=torch.arange(max(T, 1), **i32),
            sh_sorted_j=torch.zeros(max(T, 1), **i32), sh_active=torch.tensor([1, 0], **i32),
        )
        if T not in self._bufs:
            self._bufs[T] = b
        return b

    def forward(self, layer: int, x: torch.Tensor, b: Buffers | None = None, stream=None,
                combine: str = "kernel", ffn_events=None) -> Buffers:
        """Enqueue one layer on x (bf16 bits as int16/uint16-sized tensor [T][d]).

        combine="kernel": routed experts write y_e rows (y_perm), the shared
        expert y_sh, and moe_combine forms y. combine="atomic": the shared
        expert writes y directly and the routed call adds gate * y_e into it
        (moe_expert_ffn with topk_w), with no y_perm and no combine pass.
        ffn_events: a pair of CUDA events recorded around the expert calls
        (routed and shared), on the stream the layer runs on."""
        wl = self.wl
        T = x.shape[0]
        b = b or self.buffers(T)
        k, E, d, f = wl.k, wl.E, wl.d, wl.f
        native.route(x, self.Wr[layer], self.bias[layer], T, d, E, k, b.logits, b.idx, b.w, b.status, stream)
        native.permute(b.idx, T, k, E, b.counts, b.offsets, b.sorted_tok, b.sorted_j, b.inv, b.active, b.perm_ws,
                       0 if b.perm_ws is None else b.perm_ws.numel(), b.status, stream)
        native.cache_lookup(self.slot_of[layer], self.num_slots, layer, b.idx, b.w, b.offsets, b.sorted_tok,
                            b.sorted_j, T, k, E, b.sop, b.miss, b.miss_count, b.idx.numel(), b.status, stream,
                            expert_counts=self.expert_counts[layer] if self.count_experts else None)
        routed = [(self.qpools[fm], self.slot_of_fmt_all[fm][layer]) for fm in self.fmts] if self.mixed \
            else [(self.qpool, self.slot_of[layer])]
        st = torch.cuda.current_stream() if stream is None else stream
        if ffn_events:
            ffn_events[0].record(st)
        if combine == "atomic":
            native.expert_ffn(self.qpool, self.shared_slot[layer], x, T, d, f, 1, 1, b.sh_offsets, b.sh_sorted_tok,
                              b.sh_sorted_j, b.sh_active, None, b.y, b.h_sh, b.h_sh.numel(), b.status, stream)
            for pool, table in routed:
                native.expert_ffn(pool, table, x, T, d, f, E, k, b.offsets, b.sorted_tok, b.sorted_j, b.active, b.w,
                                  b.y, b.h_ws, b.h_ws.numel(), b.status, stream)
            if ffn_events:
                ffn_events[1].record(st)
            return b
        for pool, table in routed:
            native.expert_ffn(pool, table, x, T, d, f, E, k, b.offsets, b.sorted_tok, b.sorted_j, b.active, None,
                              b.y_perm, b.h_ws, b.h_ws.numel(), b.status, stream)
        native.expert_ffn(self.qpool, self.shared_slot[layer], x, T, d, f, 1, 1, b.sh_offsets, b.sh_sorted_tok,
                          b.sh_sorted_j, b.sh_active, None, b.y_sh, b.h_sh, b.h_sh.numel(), b.status, stream)
        if ffn_events:
            ffn_events[1].record(st)
        native.combine(b.y_perm, b.inv, b.w, b.sop, b.y_sh, T, k, d, b.y, stream)
        return b

    def forward_chunked_host(self, layer: int, x_host: torch.Tensor, y_host: torch.Tensor, chunk: int = 8192,
                             combine: str = "kernel") -> None:
        """A long prompt from pinned host memory to pinned host memory in chunks
        of at most `chunk` tokens, copies overlapped with the layer: chunk c+1
        is copied in on one side stream and chunk c-1's y copied out on another
        while chunk c runs on the current stream (two device buffers of each).
        x_host: pinned int16 [T][d] (bf16 bits); y_host: pinned fp32 [T][d].
        When the current stream reaches the end of what this enqueues, y_host
        holds every chunk's output."""
        wl, dev = self.wl, self.device
        T = x_host.shape[0]
        main = torch.cuda.current_stream()
        key = ("chunk_io", chunk)
        if key not in self._ws:
            self._ws[key] = {
                "h2d": torch.cuda.Stream(device=dev), "d2h": torch.cuda.Stream(device=dev),
                "x": [torch.empty((chunk, wl.d), dtype=torch.int16, device=dev) for _ in range(2)],
                "y": [torch.empty((chunk, wl.d), dtype=torch.float32, device=dev) for _ in range(2)],
            }
        io = self._ws[key]
        h2d, d2h = io["h2d"], io["d2h"]
        h2d.wait_stream(main)             # nothing is copied before the work queued so far
        d2h.wait_stream(main)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [None, None]
        ev_out = [None, None]
        last = None
        for c, c0 in enumerate(range(0, T, chunk)):
            i, n = c % 2, min(chunk, T - c0)
            with torch.cuda.stream(h2d):
                if ev_done[i] is not None:
                    h2d.wait_event(ev_done[i])       # the layer that read x buffer i is done
                io["x"][i][:n].copy_(x_host[c0:c0 + n], non_blocking=True)
                ev_in[i].record(h2d)
            main.wait_event(ev_in[i])
            if ev_out[i] is not None:
                main.wait_event(ev_out[i])           # y buffer i has been copied out
            b = dataclasses.replace(self.buffers(n), y=io["y"][i][:n])
            self.forward(layer, io["x"][i][:n], b, combine=combine)
            ev_done[i] = torch.cuda.Event()
            ev_done[i].record(main)
            with torch.cuda.stream(d2h):
                d2h.wait_event(ev_done[i])
                y_host[c0:c0 + n].copy_(io["y"][i][:n], non_blocking=True)
                ev_out[i] = torch.cuda.Event()
                ev_out[i].record(d2h)
                last = ev_out[i]
        if last is not None:
            main.wait_event(last)

    def launches(self, T: int, combine: str = "kernel") -> int:
        """Kernel launches forward() makes for T tokens (route 2, permute 1 or
        3, lookup 1, each expert call 2, or 3 on the tensor-core path, combine 1)."""
        wl = self.wl
        ffn = lambda n, fm: 3 if n >= 512 and fm == 2 else 2  # noqa: E731
        perm = 1 if native.permute_workspace_bytes(T, wl.k, wl.E) == 0 else 3
        routed = sum(ffn(T * wl.k, fm) for fm in self.fmts)
        return 2 + perm + 1 + routed + ffn(T, wl.fmt) + (1 if combine == "kernel" else 0)

    def forward_chunked(self, layer: int, x: torch.Tensor, chunk: int = 8192, y: torch.Tensor | None = None,
                        stream=None, combine: str = "kernel", ffn_events=None) -> torch.Tensor:
        """A long prompt through one layer in chunks of at most `chunk` tokens,
        back to back on one stream (each chunk is one forward(); the last may
        be shorter). Returns y fp32 [T][d] (``y`` if given). ffn_events: one
        pair of events per chunk (see forward)."""
        T = x.shape[0]
        y = torch.empty((T, self.wl.d), dtype=torch.float32, device=self.device) if y is None else y
        for i, c0 in enumerate(range(0, T, chunk)):
            n = min(chunk, T - c0)
            # the chunk's buffers, with its output rows written in place in y
            b = dataclasses.replace(self.buffers(n), y=y[c0:c0 + n])
            self.forward(layer, x[c0:c0 + n], b, stream=stream, combine=combine,
                         ffn_events=None if ffn_events is None else ffn_events[i])
        return y

    def decode_workspace(self, T: int) -> torch.Tensor:
        """Zero-filled workspace of moe_layer_decode for T tokens (kept per T)."""
        key = ("dec", T)
        if key not in self._ws:
            n = native.layer_decode_workspace_bytes(T, self.wl.k, self.wl.f, self.wl.E)
            self._ws[key] = torch.zeros(max(n, 256), dtype=torch.uint8, device=self.device)
        return self._ws[key]

    def forward_fused(self, layer: int, x: torch.Tensor, b: Buffers | None = None, stream=None,
                      outputs: bool = True) -> Buffers:
        """Enqueue one layer as a single moe_layer_decode launch (T <= 8).
        outputs=False skips the routing/permutation side outputs (only y)."""
        if self.mixed:
            raise ValueError("the one-launch decode kernel reads a single-format pool; use forward()")
        wl = self.wl
        T = x.shape[0]
        b = b or self.buffers(T)
        ws = self.decode_workspace(T)
        o = outputs
        native.layer_decode(self.qpool, self.slot_of[layer], self.L * self.R + layer, layer, x, self.Wr[layer],
                            self.bias[layer], T, wl.d, wl.f, wl.E, wl.k,
                            logits=b.logits if o else None, topk_idx=b.idx if o else None,
                            topk_w=b.w if o else None, counts=b.counts if o else None,
                            offsets=b.offsets if o else None, sorted_tok=b.sorted_tok if o else None,
                            sorted_j=b.sorted_j if o else None, inv=b.inv if o else None,
                            active=b.active if o else None, slot_of_pair=b.sop if o else None,
                            miss=b.miss if o else None, miss_count=b.miss_count if o else None,
                            miss_cap=b.idx.numel() if o else 0, y=b.y, ws=ws, ws_bytes=ws.numel(),
                            dev_status=b.status, stream=stream,
                            expert_counts=self.expert_counts[layer] if self.count_experts else None)
        return b

    def stack_buffers(self, T: int, host_misses: bool = False) -> "StackBuffers":
        """Outputs of moe_stack_decode for T tokens through all L layers (kept per
        T). With host_misses the miss records and counts live in mapped pinned
        host memory (the kernel writes them there layer by layer; see
        MissEngine), else on the device."""
        key = ("stack", T, host_misses)
        if key not in self._ws:
            wl, dev, L = self.wl, self.device, self.L
            n = max(T * wl.k, 1)
            i32 = dict(dtype=torch.int32, device=dev)
            if host_misses:
                miss = MappedHostBuffer(L * n * native.MISS_BYTES)
                count = MappedHostBuffer(L * 4)
                count.view(np.int32)[:] = -1
            else:
                miss = torch.empty(L, n * native.MISS_BYTES, dtype=torch.uint8, device=dev)
                count = torch.zeros(L, **i32)
            self._ws[key] = StackBuffers(
                T=T, idx=torch.empty(L, n, **i32), w=torch.empty(L, n, dtype=torch.float32, device=dev),
                sop=torch.empty(L, n, **i32), miss=miss, miss_count=count,
                y=torch.empty(L, max(T, 1), wl.d, dtype=torch.float32, device=dev), status=torch.zeros(1, **i32))
        return self._ws[key]

    def forward_stack(self, x: torch.Tensor, b: "StackBuffers | None" = None, stream=None) -> "StackBuffers":
        """Enqueue all L layers as one moe_stack_decode launch; x is [L][T][d]
        (bf16 bits), layer l's input in x[l]. T <= 8."""
        if self.mixed:
            raise ValueError("the stacked decode kernel reads a single-format pool; use forward()")
        wl = self.wl
        T = x.shape[1]
        b = b or self.stack_buffers(T)
        ws = self.decode_workspace(T)
        n = max(T * wl.k, 1)
        native.stack_decode(self.qpool, self.L, self.slot_of_all, self.shared_slot_all, 0, x, self.Wr_all,
                            self.bias_all, T, wl.d, wl.f, wl.E, wl.k, topk_idx=b.idx, topk_w=b.w, slot_of_pair=b.sop,
                            miss=b.miss, miss_count=b.miss_count, miss_cap=n, y=b.y, ws=ws, ws_bytes=ws.numel(),
                            dev_status=b.status, stream=stream,
                            expert_counts=self.expert_counts if self.count_experts else None)
        return b

    def stack_misses(self, b: "StackBuffers", layer: int) -> list:
        """Miss records of one layer of the last forward_stack (host copy; synchronises)."""
        cap = b.idx.shape[1]
        if isinstance(b.miss, MappedHostBuffer):
            torch.cuda.synchronize()
            n = min(int(b.miss_count.view(np.int32)[layer]), cap)
            rec = b.miss.view(MISS_DTYPE, (self.L, cap))[layer, :n].copy()
        else:
            n = min(int(b.miss_count[layer].item()), cap)
            raw = b.miss[layer, : n * native.MISS_BYTES].cpu().numpy().tobytes()
            rec = np.frombuffer(raw, dtype=MISS_DTYPE)
        return [(int(r["layer"]), int(r["expert"]), int(r["token"]), int(r["j"]), float(r["gate"])) for r in rec]

    def misses(self, b: Buffers) -> list:
        """Miss records of the last forward (host copy; synchronises)."""
        n = int(b.miss_count.item())
        raw = b.miss[: min(n, b.idx.numel()) * native.MISS_BYTES].cpu().numpy().tobytes()
        rec = np.frombuffer(raw, dtype=np.dtype([("layer", "<i4"), ("expert", "<i4"), ("token", "<i4"),
                                                 ("j", "<i4"), ("gate", "<f4")]))
        return [(int(r["layer"]), int(r["expert"]), int(r["token"]), int(r["j"]), float(r["gate"])) for r in rec]


def x_tensor(x_bits: np.ndarray, device="cuda") -> torch.Tensor:
    """bf16 bit patterns (uint16 numpy) as a device int16 tensor of the same bytes."""
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).to(device)
