"""The oracle's layer, spread over host processes (test infrastructure).

``orc.moe_layer`` at full expert size costs a dequantisation per expert and a
plain C matrix-vector product per (token, expert) pair: minutes for a
512-token prefill on one core.  ``layer_outputs`` computes exactly the same
thing from the same oracle steps -- the oracle router, then every routed
expert dequantised and applied by the oracle to the rows routed to it, then
the oracle combine -- with the (expert, rows) jobs spread over a pool of
worker processes.  The pool uses the spawn start method (a process forked
after CUDA is initialised can hang) and lives until the test session ends.
"""
from __future__ import annotations

import atexit
import multiprocessing as mp
import os

import numpy as np

from expert_cached_sparse_b200 import workloads as W

_pool = None


def pool():
    global _pool
    if _pool is None:
        n = max(1, min(16, os.cpu_count() or 1))
        _pool = mp.get_context("spawn").Pool(n)
        atexit.register(_close)
    return _pool


def _close():
    global _pool
    if _pool is not None:
        _pool.terminate()
        _pool = None


def _expert_rows(job):
    """One routed expert of one layer call on its rows: float64 [m, H]."""
    cfg, seed, key, x_rows = job
    from oracle import oracle as orc
    ew = W.gen_expert(cfg, seed, *key)
    w13, w2 = orc.dequant_expert(cfg.wfmt, ew, cfg.hidden, cfg.ffn)
    return np.stack([orc.expert_ffn(w13, w2, x) for x in x_rows])


def layer_outputs(orc, cfg: W.LayerConfig, seed: int, distinct, calls):
    """calls: [(layer, x, wg_bits, bias, tokens or None)].  For each call the
    oracle layer on those tokens: (out float64 [n, H], idx, w), as
    ``orc.moe_layer`` returns them.  Expert e of layer l has the weights of
    ``W.blob_alias(cfg, l, e, distinct)`` (the GPU tests' blob aliasing)."""
    k = cfg.top_k
    jobs, plan = [], []
    for layer, x, wg, bias, tokens in calls:
        xs = x if tokens is None else x[np.asarray(tokens)]
        _, idx, w = orc.router(xs, wg, bias, k)
        xf = orc.as_f32(xs).astype(np.float64)
        flat = idx.reshape(-1)
        parts = []
        for e in np.unique(flat):
            a = np.flatnonzero(flat == e)
            jobs.append((cfg, seed, W.blob_alias(cfg, layer, int(e), distinct), xf[a // k]))
            parts.append(a)
        plan.append((idx, w, parts))
    results = pool().map(_expert_rows, jobs, chunksize=1) if jobs else []
    out, j = [], 0
    for idx, w, parts in plan:
        y = np.empty((idx.size, cfg.hidden), np.float64)
        for a in parts:
            y[a] = results[j]
            j += 1
        out.append((orc.combine(y, w), idx, w))
    return out
