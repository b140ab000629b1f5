"""Python face of the CPU oracle (test infrastructure only).

Loads ``liboracle.so`` (built from ``moe_oracle.c`` by :func:`build`) with
ctypes and strings its steps together: route, look up / update the LRU
cache, permute, dequantise, run the SwiGLU experts, combine.  Only the test
suite, the package smoke check and the benchmark's CPU-baseline leg use it;
the CUDA library never does.  Nothing here is shared with the CUDA path
except the seeded input generators in ``expert_cached_sparse_b200.workloads``,
which draw inputs and hold none of the layer's arithmetic.

Format conversions done here are encodings only: bf16 bit patterns are
widened to float exactly.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

EV_HIT, EV_MISS, EV_EVICT, EV_MOVE = 0, 1, 2, 3
ORC_ERR_CAPACITY = -2

REC_DTYPE = np.dtype([("call", "<u4"), ("slot", "<i4"), ("layer", "<u2"), ("expert", "<u2"),
                      ("event", "u1"), ("pad", "u1", 3)])


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (single thread, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = C.CDLL(build())
        P = C.c_void_p
        i32 = C.c_int
        L.orc_e2m1.restype = C.c_double
        L.orc_e8m0.restype = C.c_double
        L.orc_e4m3.restype = C.c_double
        for f in (L.orc_e2m1, L.orc_e8m0, L.orc_e4m3):
            f.argtypes = [i32]
        L.orc_dequant_mxfp4.argtypes = [P, P, i32, i32, P]
        L.orc_dequant_nvfp4.argtypes = [P, P, C.c_float, i32, i32, P]
        L.orc_dequant_bf16.argtypes = [P, C.c_size_t, P]
        L.orc_router.argtypes = [P, P, P, i32, i32, i32, i32, P, P, P]
        L.orc_lru_create.restype = P
        L.orc_lru_create.argtypes = [i32, i32, i32]
        L.orc_lru_destroy.argtypes = [P]
        L.orc_lru_call.argtypes = [P, i32, P, i32, P, P, i32, P]
        L.orc_lru_resize.argtypes = [P, i32, P, i32, P]
        L.orc_lru_state.argtypes = [P, P, P, P]
        L.orc_lru_capacity.argtypes = [P]
        L.orc_lru_clock.argtypes = [P]
        L.orc_lru_clock.restype = C.c_uint32
        L.orc_permute.argtypes = [P, i32, i32, i32, P, P, P]
        L.orc_expert_ffn.argtypes = [P, P, i32, i32, P, P]
        L.orc_combine.argtypes = [P, P, i32, i32, i32, P]
        L.orc_act_terms.argtypes = [P, i32, i32, i32, P, P, P]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def _bf16_to_f32(b):
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def as_f32(x: np.ndarray) -> np.ndarray:
    """Activations given as float32 or as bf16 bit patterns (uint16), widened exactly."""
    return np.ascontiguousarray(x if x.dtype == np.float32 else _bf16_to_f32(x), dtype=np.float32)


# ------------------------------------------------------------------ formats
def e2m1(code: int) -> float:
    return lib().orc_e2m1(code)


def e8m0(code: int) -> float:
    return lib().orc_e8m0(code)


def e4m3(code: int) -> float:
    return lib().orc_e4m3(code)


def dequant_matrix(wfmt: int, q, scales, tensor_scale, rows: int, cols: int) -> np.ndarray:
    out = np.empty((rows, cols), np.float64)
    q = np.ascontiguousarray(q)
    if wfmt == 0:
        lib().orc_dequant_bf16(_p(q), rows * cols, _p(out))
    elif wfmt == 1:
        s = np.ascontiguousarray(scales, np.uint8)
        lib().orc_dequant_mxfp4(_p(q), _p(s), rows, cols, _p(out))
    elif wfmt == 2:
        s = np.ascontiguousarray(scales, np.uint8)
        lib().orc_dequant_nvfp4(_p(q), _p(s), float(tensor_scale), rows, cols, _p(out))
    else:
        raise ValueError(wfmt)
    return out


def dequant_expert(wfmt: int, ew, hidden: int, ffn: int):
    """(W13 [2F][H], W2 [H][F]) as float64."""
    w13 = dequant_matrix(wfmt, ew.w13, ew.w13_scales, ew.tensor_scales[0], 2 * ffn, hidden)
    w2 = dequant_matrix(wfmt, ew.w2, ew.w2_scales, ew.tensor_scales[1], hidden, ffn)
    return w13, w2


# ------------------------------------------------------------------ activation terms
def act_terms(x, wfmt: int, terms: int):
    """Rows of activations (float32, or bf16 bits) as sums of E2M1 terms.

    Returns (codes uint8 [n, T, K], scales uint8 [n, T, K/vs], p int32 [n]):
    row i is approximately 2^-p[i] * sum_t e2m1(codes[i, t]) * scale(scales[i, t]).
    """
    xf = as_f32(np.atleast_2d(x))
    n, k = xf.shape
    vs = 32 if wfmt == 1 else 16
    codes = np.empty((n, terms, k), np.uint8)
    scales = np.empty((n, terms, k // vs), np.uint8)
    p = np.empty(n, np.int32)
    pi = C.c_int(0)
    for i in range(n):
        row = np.ascontiguousarray(xf[i])
        c = np.empty((terms, k), np.uint8)
        s = np.empty((terms, k // vs), np.uint8)
        rc = lib().orc_act_terms(_p(row), k, wfmt, terms, _p(c), _p(s), C.byref(pi))
        if rc:
            raise ValueError(f"orc_act_terms: {rc}")
        codes[i], scales[i], p[i] = c, s, pi.value
    return codes, scales, p


# ------------------------------------------------------------------ router
def router(x, wg_bits, bias, k: int):
    """(logits f32 [n,E], idx i32 [n,k], w f64 [n,k]) for activations x."""
    xf = as_f32(x)
    wf = _bf16_to_f32(wg_bits)
    n, h = xf.shape
    e = wf.shape[0]
    logits = np.empty((n, e), np.float32)
    idx = np.empty((n, k), np.int32)
    w = np.empty((n, k), np.float64)
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    rc = lib().orc_router(_p(xf), _p(wf), None if b is None else _p(b), n, h, e, k,
                          _p(logits), _p(idx), _p(w))
    if rc:
        raise ValueError(f"orc_router: {rc}")
    return logits, idx, w


# ------------------------------------------------------------------ LRU
class Lru:
    """The shared (layer, expert) LRU slot cache."""

    def __init__(self, layers: int, experts: int, capacity: int):
        self.layers, self.experts = layers, experts
        self._h = lib().orc_lru_create(layers, experts, capacity)
        if not self._h:
            raise ValueError("bad LRU shape")

    def __del__(self):
        if getattr(self, "_h", None):
            lib().orc_lru_destroy(self._h)
            self._h = None

    @property
    def capacity(self) -> int:
        return lib().orc_lru_capacity(self._h)

    @property
    def clock(self) -> int:
        return lib().orc_lru_clock(self._h)

    def call(self, layer: int, idx):
        """-> (status, records structured array, slot_of_expert [E])."""
        idx = np.ascontiguousarray(np.asarray(idx).reshape(-1), np.int32)
        cap = 2 * idx.size + 1
        out = np.zeros(cap, REC_DTYPE)
        slots = np.full(self.experts, -1, np.int32)
        n = C.c_int(0)
        rc = lib().orc_lru_call(self._h, layer, _p(idx), idx.size, _p(slots), _p(out), cap,
                                C.byref(n))
        return rc, out[: n.value].copy(), slots

    def resize(self, new_capacity: int):
        cap = 2 * max(self.capacity, new_capacity) + 1
        out = np.zeros(cap, REC_DTYPE)
        n = C.c_int(0)
        rc = lib().orc_lru_resize(self._h, new_capacity, _p(out), cap, C.byref(n))
        return rc, out[: n.value].copy()

    def state(self):
        slot_of = np.empty(self.layers * self.experts, np.int32)
        key_of = np.empty(self.capacity, np.int32)
        stamp = np.empty(self.capacity, np.uint64)
        lib().orc_lru_state(self._h, _p(slot_of), _p(key_of), _p(stamp))
        return slot_of, key_of, stamp


# ------------------------------------------------------------------ permute
def permute(idx, experts: int):
    idx = np.ascontiguousarray(idx, np.int32)
    n, k = idx.shape
    offsets = np.empty(experts + 1, np.int32)
    row_of = np.empty(n * k, np.int32)
    assign_of = np.empty(n * k, np.int32)
    rc = lib().orc_permute(_p(idx), n, experts, k, _p(offsets), _p(row_of), _p(assign_of))
    if rc:
        raise ValueError(f"orc_permute: {rc}")
    return offsets, row_of, assign_of


# ------------------------------------------------------------------ FFN + combine
def expert_ffn(w13, w2, x) -> np.ndarray:
    w13 = np.ascontiguousarray(w13, np.float64)
    w2 = np.ascontiguousarray(w2, np.float64)
    h = w2.shape[0]
    f = w2.shape[1]
    xv = np.ascontiguousarray(x, np.float64)
    y = np.empty(h, np.float64)
    lib().orc_expert_ffn(_p(w13), _p(w2), h, f, _p(xv), _p(y))
    return y


def combine(y, w) -> np.ndarray:
    """y [n*k, H] in assignment order, w [n,k] -> out [n,H] (float64)."""
    y = np.ascontiguousarray(y, np.float64)
    w = np.ascontiguousarray(w, np.float64)
    n, k = w.shape
    h = y.shape[1]
    out = np.empty((n, h), np.float64)
    lib().orc_combine(_p(y), _p(w), n, k, h, _p(out))
    return out


def moe_layer(x, wg_bits, bias, k: int, wfmt: int, hidden: int, ffn: int, expert_fn,
              tokens=None):
    """The whole layer for the chosen tokens (all by default).

    expert_fn(e) returns the canonical weights of expert e.  Returns
    (out [len(tokens), H] float64, idx, w, logits) for those tokens.  The
    cache does not change what the layer computes, so it does not appear
    here; cache behaviour is checked through :class:`Lru`.
    """
    xs = x if tokens is None else x[np.asarray(tokens)]
    logits, idx, w = router(xs, wg_bits, bias, k)
    xf = as_f32(xs).astype(np.float64)
    n = xs.shape[0]
    y = np.empty((n * k, hidden), np.float64)
    for e in np.unique(idx):
        w13, w2 = dequant_expert(wfmt, expert_fn(int(e)), hidden, ffn)
        for a in np.flatnonzero(idx.reshape(-1) == e):
            y[a] = expert_ffn(w13, w2, xf[a // k])
    return combine(y, w), idx, w, logits
