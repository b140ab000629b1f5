"""Python face of the C ABI: the same entry points, argument marshalling only.

Device buffers are torch CUDA tensors, host buffers numpy arrays or pinned
torch tensors, streams torch.cuda.Stream.  Each function raises MoeError on a
non-zero status.  Every computation happens inside libmoe.so.
"""
from __future__ import annotations

import ctypes as C

import numpy as np
import torch

from . import _lib as L
from ._lib import MoeError, check, ptr, stream_handle  # noqa: F401

DT_F32, DT_BF16 = L.DT_F32, L.DT_BF16
W_BF16, W_MXFP4, W_NVFP4 = L.W_BF16, L.W_MXFP4, L.W_NVFP4


def _dt(t) -> int:
    if t.dtype == torch.float32:
        return DT_F32
    if t.dtype in (torch.bfloat16, torch.int16, torch.uint16):
        return DT_BF16
    raise TypeError(f"activations must be float32 or bf16, got {t.dtype}")


def make_shape(layers, experts, hidden, ffn, top_k, wfmt) -> L.MoeShape:
    return L.shape(layers, experts, hidden, ffn, top_k, wfmt)


def shape_of(cfg) -> L.MoeShape:
    """Shape of a workloads.LayerConfig."""
    return make_shape(cfg.layers, cfg.experts, cfg.hidden, cfg.ffn, cfg.top_k, cfg.wfmt)


# ------------------------------------------------------------------ sizes
def moe_slot_bytes(shape) -> int:
    return L.lib.moe_slot_bytes(C.byref(shape))


def moe_cache_meta_bytes(shape, capacity, trace_capacity) -> int:
    return L.lib.moe_cache_meta_bytes(C.byref(shape), capacity, trace_capacity)


def moe_permute_workspace_bytes(n, experts, top_k) -> int:
    return L.lib.moe_permute_workspace_bytes(n, experts, top_k)


def moe_ffn_workspace_bytes(shape, rows) -> int:
    return L.lib.moe_ffn_workspace_bytes(C.byref(shape), rows)


def moe_layer_workspace_bytes(shape, n) -> int:
    return L.lib.moe_layer_workspace_bytes(C.byref(shape), n)


# ------------------------------------------------------------------ packing (host)
def moe_pack_expert(shape, ew, out: np.ndarray | None = None) -> np.ndarray:
    """Pack one workloads.ExpertWeights into a slot blob (uint8 numpy array or `out`)."""
    nb = moe_slot_bytes(shape)
    if out is None:
        out = np.empty(nb, np.uint8)
    w13 = np.ascontiguousarray(ew.w13)
    w2 = np.ascontiguousarray(ew.w2)
    s13 = None if ew.w13_scales is None else np.ascontiguousarray(ew.w13_scales, np.uint8)
    s2 = None if ew.w2_scales is None else np.ascontiguousarray(ew.w2_scales, np.uint8)
    ts = np.ascontiguousarray(ew.tensor_scales, np.float32)
    rc = L.lib.moe_pack_expert(C.byref(shape), ptr(w13), ptr(s13), ptr(w2), ptr(s2), ptr(ts), ptr(out))
    check("moe_pack_expert", rc)
    return out


# ------------------------------------------------------------------ steps
def moe_router_topk(x, wg, bias, n, hidden, experts, k, logits, topk_idx, topk_w, stream=None):
    rc = L.lib.moe_router_topk(ptr(x), _dt(x), ptr(wg), ptr(bias), n, hidden, experts, k, ptr(logits),
                               ptr(topk_idx), ptr(topk_w), stream_handle(stream))
    check("moe_router_topk", rc)


def moe_permute(topk_idx, n, experts, k, x, hidden, offsets, row_of, assign_of, x_perm, ws, stream=None):
    rc = L.lib.moe_permute(ptr(topk_idx), n, experts, k, ptr(x), _dt(x), hidden, ptr(offsets), ptr(row_of),
                           ptr(assign_of), ptr(x_perm), ptr(ws), ws.numel() * ws.element_size(),
                           stream_handle(stream))
    check("moe_permute", rc)


def moe_permute_noalloc(topk_idx, n, experts, k, x, hidden, offsets, row_of, assign_of, x_perm, stream=None):
    """moe_permute with the library's static scratch instead of a workspace (see include/moe.h)."""
    rc = L.lib.moe_permute_noalloc(ptr(topk_idx), n, experts, k, ptr(x), _dt(x), hidden, ptr(offsets), ptr(row_of),
                                   ptr(assign_of), ptr(x_perm), stream_handle(stream))
    check("moe_permute_noalloc", rc)


def moe_grouped_ffn(shape, pool, pool_slots, slot_of, offsets, x_perm, rows, y_perm, ws, stream=None):
    rc = L.lib.moe_grouped_ffn(C.byref(shape), ptr(pool), pool_slots, ptr(slot_of), ptr(offsets), ptr(x_perm), rows,
                               ptr(y_perm), ptr(ws), ws.numel() * ws.element_size(), stream_handle(stream))
    check("moe_grouped_ffn", rc)


def moe_act_terms(x, rows, K, wfmt, terms, codes, scales, row_exp, stream=None):
    """E2M1 term encoding of activation rows (the FP4 path's operand encoding):
    codes uint8 [rows, terms, K], scales uint8 [rows, terms, K/vs], row_exp int32 [rows]."""
    rc = L.lib.moe_act_terms(ptr(x), _dt(x), rows, K, wfmt, terms, ptr(codes), ptr(scales), ptr(row_exp),
                             stream_handle(stream))
    check("moe_act_terms", rc)


def moe_combine(y_perm, row_of, topk_w, n, k, hidden, out, stream=None):
    rc = L.lib.moe_combine(ptr(y_perm), ptr(row_of), ptr(topk_w), n, k, hidden, ptr(out), _dt(out),
                           stream_handle(stream))
    check("moe_combine", rc)


# ------------------------------------------------------------------ cache
class MoeCache:
    """A moe_cache plus the device buffers it lives in (allocated here by torch).

    host_blobs: list of L*E pinned uint8 tensors / numpy arrays (entries may
    repeat); the object keeps references so they outlive the cache.
    """

    def __init__(self, shape, capacity: int, host_blobs, trace_capacity: int = 1 << 16,
                 device="cuda", stream=None):
        self.shape = shape
        self.slot_bytes = moe_slot_bytes(shape)
        self.trace_capacity = trace_capacity
        mb = moe_cache_meta_bytes(shape, capacity, trace_capacity)
        if mb == 0 or self.slot_bytes == 0:
            raise MoeError("moe_cache_meta_bytes", L.MOE_ERR_INVALID_ARG)
        self.meta = torch.empty(mb, dtype=torch.uint8, device=device)
        self.pool = torch.empty(capacity * self.slot_bytes, dtype=torch.uint8, device=device)
        self._blobs = list(host_blobs)
        arr = (C.c_void_p * len(self._blobs))(*[ptr(b) for b in self._blobs])
        self._arr = arr
        h = C.c_void_p()
        rc = L.lib.moe_cache_create(C.byref(shape), ptr(self.meta), mb, ptr(self.pool), capacity,
                                    trace_capacity, arr, stream_handle(stream), C.byref(h))
        check("moe_cache_create", rc)
        self.handle = h

    @property
    def capacity(self) -> int:
        return L.lib.moe_cache_capacity(self.handle)

    def lookup_update(self, layer, idx, slot_of=None, stream=None, copy_stream=None):
        rc = L.lib.moe_cache_lookup_update(self.handle, layer, ptr(idx), idx.numel(), ptr(slot_of),
                                           stream_handle(stream), stream_handle(copy_stream))
        check("moe_cache_lookup_update", rc)

    def resize(self, new_capacity: int, stream=None, in_place: bool = False):
        mb = moe_cache_meta_bytes(self.shape, new_capacity, self.trace_capacity)
        if in_place and new_capacity <= self.capacity and mb <= self.meta.numel():
            meta, pool = self.meta, self.pool
        else:
            meta = torch.empty(mb, dtype=torch.uint8, device=self.meta.device)
            pool = torch.empty(new_capacity * self.slot_bytes, dtype=torch.uint8, device=self.pool.device)
        rc = L.lib.moe_cache_resize(self.handle, ptr(meta), meta.numel(), ptr(pool), new_capacity,
                                    stream_handle(stream))
        check("moe_cache_resize", rc)
        self.meta, self.pool = meta, pool

    def set_fill_mode(self, mode: int, stream=None):
        """L.FILL_HOST (host-issued DMA copies) or L.FILL_DEVICE (zero-copy fill kernel)."""
        check("moe_cache_set_fill_mode", L.lib.moe_cache_set_fill_mode(self.handle, mode, stream_handle(stream)))

    @property
    def fill_mode(self) -> int:
        return L.lib.moe_cache_fill_mode(self.handle)

    def device_status(self, clear: bool = False) -> int:
        """First error a lookup kernel recorded since the last clear (0 if none)."""
        rc = L.lib.moe_cache_device_status(self.handle, 1 if clear else 0)
        if rc in (L.MOE_ERR_CUDA,):
            raise MoeError("moe_cache_device_status", rc)
        return rc

    def read_trace(self, cap: int | None = None) -> np.ndarray:
        cap = self.trace_capacity if cap is None else cap
        buf = np.zeros(cap, L.TRACE_DTYPE)
        n = C.c_size_t(0)
        check("moe_cache_read_trace", L.lib.moe_cache_read_trace(self.handle, ptr(buf), cap, C.byref(n)))
        return buf[: n.value].copy()

    def stats(self) -> dict:
        s = L.MoeStats()
        check("moe_cache_get_stats", L.lib.moe_cache_get_stats(self.handle, C.byref(s)))
        return {name: getattr(s, name) for name, _ in L.MoeStats._fields_}

    def snapshot(self):
        nk = self.shape.layers * self.shape.experts
        c = self.capacity
        slot_of = np.empty(nk, np.int32)
        key_of = np.empty(c, np.int32)
        stamp = np.empty(c, np.uint64)
        check("moe_cache_snapshot", L.lib.moe_cache_snapshot(self.handle, ptr(slot_of), ptr(key_of), ptr(stamp)))
        return slot_of, key_of, stamp

    def close(self):
        if getattr(self, "handle", None):
            L.lib.moe_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_layer_forward(cache: MoeCache, layer, x, wg, bias, out, ws, stream=None, copy_stream=None,
                      topk_idx_out=None, topk_w_out=None):
    n = x.shape[0]
    rc = L.lib.moe_layer_forward(cache.handle, layer, ptr(x), _dt(x), ptr(wg), ptr(bias), n, ptr(out), ptr(ws),
                                 ws.numel() * ws.element_size(), stream_handle(stream),
                                 stream_handle(copy_stream), ptr(topk_idx_out), ptr(topk_w_out))
    check("moe_layer_forward", rc)


def moe_prefill_workspace_bytes(shape, n) -> int:
    return L.lib.moe_prefill_workspace_bytes(C.byref(shape), n)


def moe_prefill_forward(cache: MoeCache, layer0, xs, wgs, biases, outs, ws, stream=None, copy_stream=None,
                        topk_idx_out=None):
    """Layers layer0 .. layer0+len(xs)-1 over one prompt; xs / wgs / biases / outs are per-layer
    device tensors (biases may be None or hold None; outs[i] may be xs[i+1])."""
    nl = len(xs)
    if not (len(wgs) == len(outs) == nl) or (biases is not None and len(biases) != nl):
        raise ValueError("per-layer lists of different lengths")
    n = xs[0].shape[0] if nl else 0
    arr = lambda ts: (C.c_void_p * max(1, nl))(*[ptr(t) for t in ts])
    xa, wa, oa = arr(xs), arr(wgs), arr(outs)
    ba = None if biases is None else arr(biases)
    rc = L.lib.moe_prefill_forward(cache.handle, layer0, nl, xa, _dt(xs[0]) if nl else 0, wa, ba, n, oa, ptr(ws),
                                   ws.numel() * ws.element_size(), stream_handle(stream), stream_handle(copy_stream),
                                   ptr(topk_idx_out))
    check("moe_prefill_forward", rc)


# ------------------------------------------------------------------ testing hooks
def moe_test_set_wait(cycles: int, withhold: bool = False) -> None:
    """Bounded-wait limit (SM cycles, 0 = default) and stage withholding of later FFN launches."""
    check("moe_test_set_wait", L.lib.moe_test_set_wait(int(cycles), 1 if withhold else 0))


def moe_get_device_error(clear: bool = False) -> int:
    rc = L.lib.moe_get_device_error(1 if clear else 0)
    if rc == L.MOE_ERR_CUDA:
        raise MoeError("moe_get_device_error", rc)
    return rc


# ------------------------------------------------------------------ profiling
def moe_profile_enable(timing: bool) -> None:
    check("moe_profile_enable", L.lib.moe_profile_enable(1 if timing else 0))


def moe_profile_read(reset: bool = False) -> dict:
    """{kind: {"launches", "timed", "ms"}} for router/lookup/permute/ffn/combine/fill."""
    arr = (L.MoeProf * len(L.PROF_KINDS))()
    check("moe_profile_read", L.lib.moe_profile_read(arr, len(L.PROF_KINDS), 1 if reset else 0))
    return {k: {"launches": arr[i].launches, "timed": arr[i].timed, "ms": arr[i].ms}
            for i, k in enumerate(L.PROF_KINDS)}
