"""ctypes binding of libmoe.so (include/moe.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  Device buffers are torch CUDA tensors (or raw integer
addresses), host buffers numpy arrays, streams torch.cuda.Stream objects (or
raw handles).  If libmoe.so is missing this module raises on import; there
is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_CAPACITY = -2
MOE_ERR_CUDA = -3
MOE_ERR_FILL = -4
MOE_ERR_TIMEOUT = -5
MOE_ERR_UNSUPPORTED = -6
MOE_ERR_STATE = -7
DT_F32, DT_BF16 = 0, 1
W_BF16, W_MXFP4, W_NVFP4 = 0, 1, 2
FILL_HOST, FILL_DEVICE = 0, 1

EXPORTS = [
    "moe_status_str", "moe_version", "moe_slot_bytes", "moe_cache_meta_bytes",
    "moe_permute_workspace_bytes", "moe_ffn_workspace_bytes", "moe_layer_workspace_bytes",
    "moe_pack_expert", "moe_cache_create", "moe_cache_lookup_update", "moe_cache_resize",
    "moe_cache_read_trace", "moe_cache_get_stats", "moe_cache_snapshot", "moe_cache_capacity",
    "moe_cache_destroy", "moe_router_topk", "moe_permute", "moe_grouped_ffn", "moe_combine",
    "moe_layer_forward", "moe_profile_enable", "moe_profile_read", "moe_get_device_error",
    "moe_permute_noalloc", "moe_act_terms", "moe_cache_set_fill_mode", "moe_cache_fill_mode",
    "moe_cache_device_status", "moe_test_set_wait", "moe_prefill_workspace_bytes", "moe_prefill_forward",
]
PROF_KINDS = ["router", "lookup", "permute", "ffn", "combine", "fill"]

TRACE_DTYPE = np.dtype([("call", "<u4"), ("slot", "<i4"), ("layer", "<u2"), ("expert", "<u2"),
                        ("event", "u1"), ("pad", "u1", 3)])


class MoeShape(C.Structure):
    _fields_ = [("layers", C.c_int32), ("experts", C.c_int32), ("hidden", C.c_int32),
                ("ffn", C.c_int32), ("top_k", C.c_int32), ("wfmt", C.c_int32)]


class MoeStats(C.Structure):
    _fields_ = [(n, C.c_uint64) for n in ("lookups", "hits", "misses", "evictions", "fill_bytes",
                                           "host_syncs", "trace_dropped")]


class MoeProf(C.Structure):
    _fields_ = [("launches", C.c_uint64), ("timed", C.c_uint64), ("ms", C.c_double)]


class MoeError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn}: {code} ({status_str(code)})")
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmoe.so not built at {LIB_PATH}: run expert_cached_sparse_b200.build.build()")
    L = C.CDLL(LIB_PATH)
    P, I32, SZ = C.c_void_p, C.c_int32, C.c_size_t
    SP = C.POINTER(MoeShape)
    sig = {
        "moe_status_str": (C.c_char_p, [C.c_int]),
        "moe_version": (C.c_int, []),
        "moe_slot_bytes": (SZ, [SP]),
        "moe_cache_meta_bytes": (SZ, [SP, I32, I32]),
        "moe_permute_workspace_bytes": (SZ, [I32, I32, I32]),
        "moe_ffn_workspace_bytes": (SZ, [SP, I32]),
        "moe_layer_workspace_bytes": (SZ, [SP, I32]),
        "moe_pack_expert": (C.c_int, [SP, P, P, P, P, P, P]),
        "moe_cache_create": (C.c_int, [SP, P, SZ, P, I32, I32, P, P, C.POINTER(P)]),
        "moe_cache_lookup_update": (C.c_int, [P, I32, P, I32, P, P, P]),
        "moe_cache_resize": (C.c_int, [P, P, SZ, P, I32, P]),
        "moe_cache_read_trace": (C.c_int, [P, P, SZ, C.POINTER(SZ)]),
        "moe_cache_get_stats": (C.c_int, [P, C.POINTER(MoeStats)]),
        "moe_cache_snapshot": (C.c_int, [P, P, P, P]),
        "moe_cache_capacity": (I32, [P]),
        "moe_cache_destroy": (C.c_int, [P]),
        "moe_router_topk": (C.c_int, [P, I32, P, P, I32, I32, I32, I32, P, P, P, P]),
        "moe_permute": (C.c_int, [P, I32, I32, I32, P, I32, I32, P, P, P, P, P, SZ, P]),
        "moe_permute_noalloc": (C.c_int, [P, I32, I32, I32, P, I32, I32, P, P, P, P, P]),
        "moe_grouped_ffn": (C.c_int, [SP, P, I32, P, P, P, I32, P, P, SZ, P]),
        "moe_combine": (C.c_int, [P, P, P, I32, I32, I32, P, I32, P]),
        "moe_layer_forward": (C.c_int, [P, I32, P, I32, P, P, I32, P, P, SZ, P, P, P, P]),
        "moe_profile_enable": (C.c_int, [C.c_int]),
        "moe_profile_read": (C.c_int, [C.POINTER(MoeProf), C.c_int, C.c_int]),
        "moe_get_device_error": (C.c_int, [C.c_int]),
        "moe_act_terms": (C.c_int, [P, I32, I32, I32, I32, I32, P, P, P, P]),
        "moe_cache_set_fill_mode": (C.c_int, [P, I32, P]),
        "moe_cache_fill_mode": (I32, [P]),
        "moe_cache_device_status": (C.c_int, [P, I32]),
        "moe_test_set_wait": (C.c_int, [C.c_int64, I32]),
        "moe_prefill_workspace_bytes": (SZ, [SP, I32]),
        "moe_prefill_forward": (C.c_int, [P, I32, I32, P, I32, P, P, I32, P, P, SZ, P, P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


lib = _load()


def status_str(code: int) -> str:
    return lib.moe_status_str(int(code)).decode()


def check(fn: str, code: int) -> None:
    if code != MOE_OK:
        raise MoeError(fn, code)


def ptr(t) -> int | None:
    """Device or host address of a torch tensor / numpy array / int; None for None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def stream_handle(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def shape(layers, experts, hidden, ffn, top_k, wfmt) -> MoeShape:
    return MoeShape(layers, experts, hidden, ffn, top_k, wfmt)
