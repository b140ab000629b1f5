"""Shared helpers for the GPU parity tests: device transfers, tolerances and a
layer set-up that packs seeded experts into pinned host blobs."""
from __future__ import annotations

import numpy as np
import torch

from expert_cached_sparse_b200 import api as A
from expert_cached_sparse_b200 import workloads as W

# Layer outputs and router weights: relative L2 error against the fp64 oracle
# must stay within 2e-2 (bf16 / FP4 arithmetic against the exact reference).
# Expected error is about 3e-3 (bf16 rounding of x_perm, h and y), so a
# tighter alarm catches regressions that still pass the contract.
TOL_REL_L2 = 2e-2
ALARM_REL_L2 = 6e-3


def rel_l2(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    """numpy -> device tensor; uint16 arrays are taken as bf16 bit patterns."""
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def host(t: torch.Tensor) -> np.ndarray:
    """device tensor -> numpy; bf16 becomes float64 (exact)."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.double().numpy()
    return t.numpy()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


class Layer:
    """Seeded weights of one workload: router per layer, packed experts in pinned host memory."""

    def __init__(self, cfg: W.LayerConfig, seed: int = 0, distinct: int | None = None):
        self.cfg, self.seed, self.distinct = cfg, seed, distinct
        self.shape = A.shape_of(cfg)
        self._experts = {}
        self._blobs = {}

    def expert(self, layer: int, e: int) -> W.ExpertWeights:
        key = W.blob_alias(self.cfg, layer, e, self.distinct)
        if key not in self._experts:
            self._experts[key] = W.gen_expert(self.cfg, self.seed, *key)
        return self._experts[key]

    def blob(self, layer: int, e: int) -> torch.Tensor:
        key = W.blob_alias(self.cfg, layer, e, self.distinct)
        if key not in self._blobs:
            b = torch.empty(A.moe_slot_bytes(self.shape), dtype=torch.uint8, pin_memory=True)
            A.moe_pack_expert(self.shape, self.expert(*key), out=b.numpy())
            self._blobs[key] = b
        return self._blobs[key]

    def all_blobs(self):
        c = self.cfg
        return [self.blob(l, e) for l in range(c.layers) for e in range(c.experts)]

    def drop_expert_arrays(self):
        self._experts.clear()


def make_cache(layer: Layer, capacity: int | None = None, trace_capacity: int = 1 << 18,
               stream=None) -> A.MoeCache:
    c = layer.cfg
    return A.MoeCache(layer.shape, capacity or c.capacity, layer.all_blobs(), trace_capacity=trace_capacity,
                      stream=stream)


def preload(cache: A.MoeCache, cfg: W.LayerConfig, stream=None, copy_stream=None):
    """Full residency: one lookup per layer asking for every expert, ascending."""
    idx = torch.arange(cfg.experts, dtype=torch.int32, device="cuda")
    for l in range(cfg.layers):
        cache.lookup_update(l, idx, stream=stream, copy_stream=copy_stream)
    torch.cuda.synchronize()


def trace_rows(recs) -> list[tuple]:
    return [(int(r["call"]), int(r["event"]), int(r["layer"]), int(r["expert"]), int(r["slot"])) for r in recs]


def oracle_route_trace(orc, cfg: W.LayerConfig, steps: int, prefill_tokens: int):
    """The routing of the placement study's trace (the inputs and biases that
    ``policy_study.route_trace`` feeds the GPU router), computed by the oracle
    router: (decode trace [(layer, ids)] step-major, prefill trace)."""
    E = cfg.experts
    per_layer, prefill = {}, []
    for l in range(cfg.layers):
        wg = W.gen_wg(cfg, 0, l)
        epochs = (steps + cfg.drift_every - 1) // cfg.drift_every if cfg.drift_every else 1
        rows = []
        for ep in range(epochs):
            s0 = ep * cfg.drift_every if cfg.drift_every else 0
            n = min(steps, s0 + (cfg.drift_every or steps)) - s0
            x = np.concatenate([W.gen_x(cfg, 0, 1, "policy-decode", l, s) for s in range(s0, s0 + n)])
            _, idx, _ = orc.router(x, wg, W.gen_bias(cfg, 0, l, ep), cfg.top_k)
            rows.append(idx)
        per_layer[l] = np.concatenate(rows)[:steps]
        x = W.gen_x(cfg, 0, prefill_tokens, "policy-prefill", l)
        _, idx, _ = orc.router(x, wg, W.gen_bias(cfg, 0, l, 0), cfg.top_k)
        prefill.append((l, idx))
    assert all(per_layer[l].shape == (steps, cfg.top_k) and per_layer[l].max() < E for l in per_layer)
    decode = [(l, per_layer[l][s]) for s in range(steps) for l in range(cfg.layers)]
    return decode, prefill
