"""Seeded synthetic inputs for the routed MoE layer.

This module only *draws* inputs: activations, router matrices and biases,
expert weights in the canonical (unpacked) layout, and routing-drift
permutations.  It holds none of the layer's arithmetic, so both the CUDA path
and the CPU oracle can take their inputs from here without sharing any of the
computation.

Every named tensor gets its own numpy PCG64 stream, derived from the run seed
and the tensor's name, so generation order never changes a value.

Workload shapes follow the five layer configurations the FreeToken pages talk
about: the 6-of-256 DeepSeek-V4-Flash expert layout ("Como gestiona FreeToken
la memoria MoE"), the MXFP4 / NVFP4 / BF16 precisions ("Formatos compatibles,
hardware y perfil de rendimiento"), and the shared cross-layer LRU cache over
(layer, expert) entries ("Como funciona la jerarquia de memoria MoE").
"""
from __future__ import annotations

import dataclasses
import zlib

import numpy as np

# Weight formats (values match moe_wfmt in include/moe.h).
W_BF16 = 0
W_MXFP4 = 1
W_NVFP4 = 2
FMT_NAMES = {W_BF16: "bf16", W_MXFP4: "mxfp4", W_NVFP4: "nvfp4"}


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    layers: int
    experts: int
    hidden: int
    ffn: int
    top_k: int
    wfmt: int
    x_dtype: str            # "f32" or "bf16"
    capacity: int           # expert slots in the GPU cache
    zipf_s: float | None    # None: no router bias (uniform routing)
    preload: bool           # every expert of every layer resident before timing
    drift_every: int = 0    # steps between routing drifts (0: none)
    drift_frac: float = 0.0


# The five workloads.  Sizes are the ones the layer is benchmarked at.
TINY = LayerConfig("tiny-e8-top2-h256-f512-bf16", 1, 8, 256, 512, 2, W_BF16, "f32", 8, None, True)
DS_DECODE = LayerConfig("dsv4flash-e256-top6-h4096-f2048-mxfp4-decode", 1, 256, 4096, 2048, 6,
                        W_MXFP4, "bf16", 64, 1.1, False)
DS_PREFILL = LayerConfig("dsv4flash-e256-top6-h4096-f2048-mxfp4-prefill", 1, 256, 4096, 2048, 6,
                         W_MXFP4, "bf16", 256, 0.8, True)
QWEN_BF16 = LayerConfig("qwen3-30b-a3b-e128-top8-h2048-f768-bf16", 1, 128, 2048, 768, 8,
                        W_BF16, "bf16", 128, None, True)
TRACE40 = LayerConfig("trace-l40-e256-top6-h4096-f2048-nvfp4", 40, 256, 4096, 2048, 6,
                      W_NVFP4, "bf16", 1024, 1.0, False, drift_every=32, drift_frac=0.1)

CONFIGS = {c.name: c for c in (TINY, DS_DECODE, DS_PREFILL, QWEN_BF16, TRACE40)}


def scaled(cfg: LayerConfig, **kw) -> LayerConfig:
    """A copy of cfg with some fields replaced (smaller parity cases)."""
    return dataclasses.replace(cfg, **kw)


def rng(seed: int, *name) -> np.random.Generator:
    """Independent PCG64 stream for one named tensor."""
    key = "/".join(str(p) for p in name).encode()
    ss = np.random.SeedSequence(entropy=int(seed), spawn_key=(zlib.crc32(key),))
    return np.random.Generator(np.random.PCG64(ss))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest even (input encoding only)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float32 (exact widening)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------
# activations and router
# --------------------------------------------------------------------------
def gen_x(cfg: LayerConfig, seed: int, n: int, *tag) -> np.ndarray:
    """Token activations ~N(0,1): float32 [n,H] or bf16 bits uint16 [n,H]."""
    x = rng(seed, "x", cfg.name, n, *tag).standard_normal((n, cfg.hidden), dtype=np.float32)
    return x if cfg.x_dtype == "f32" else f32_to_bf16_bits(x)


def gen_wg(cfg: LayerConfig, seed: int, layer: int) -> np.ndarray:
    """Router gate matrix Wg [E,H] as bf16 bits, entries ~N(0, 0.02)."""
    g = rng(seed, "wg", cfg.name, layer).standard_normal((cfg.experts, cfg.hidden), dtype=np.float32)
    return f32_to_bf16_bits(g * np.float32(0.02))


def zipf_rank_perm(cfg: LayerConfig, seed: int, layer: int, epoch: int = 0) -> np.ndarray:
    """perm[r] = expert holding popularity rank r (0-based) in drift epoch `epoch`.

    Epoch 0 is a seeded permutation.  Each later epoch re-shuffles the ranks of
    round(drift_frac * E) randomly chosen rank positions among themselves.
    """
    perm = rng(seed, "zipf-perm", cfg.name, layer).permutation(cfg.experts)
    m = int(round(cfg.drift_frac * cfg.experts))
    for ep in range(1, epoch + 1):
        g = rng(seed, "zipf-drift", cfg.name, layer, ep)
        pos = np.sort(g.choice(cfg.experts, size=m, replace=False))
        perm[pos] = perm[pos][g.permutation(m)]
    return perm


def gen_bias(cfg: LayerConfig, seed: int, layer: int, epoch: int = 0):
    """Router bias b[E] (float32) that tilts routing toward a Zipf(s) popularity law.

    b[perm[r]] = ln p_r with p_r proportional to (r+1)^-s.  None when the
    workload routes uniformly (no bias).
    """
    if cfg.zipf_s is None:
        return None
    r = np.arange(1, cfg.experts + 1, dtype=np.float64)
    logp = -cfg.zipf_s * np.log(r)
    logp -= np.log(np.exp(logp).sum())
    b = np.empty(cfg.experts, dtype=np.float32)
    b[zipf_rank_perm(cfg, seed, layer, epoch)] = logp.astype(np.float32)
    return b


def drift_epoch(cfg: LayerConfig, step: int) -> int:
    return step // cfg.drift_every if cfg.drift_every else 0


# --------------------------------------------------------------------------
# expert weights, canonical layout
# --------------------------------------------------------------------------
@dataclasses.dataclass
class ExpertWeights:
    """One expert in the canonical layout.

    w13: [2F][H] rows 0..F-1 gate (W1), rows F..2F-1 up (W3).
    w2:  [H][F].
    FP4 formats: two E2M1 codes per byte along a row, the even column in the
    low nibble; scales[rows][cols/32] E8M0 (MXFP4) or [rows][cols/16] E4M3
    (NVFP4); tensor_scales = (s13, s2) float32 (NVFP4; 1.0 otherwise).
    BF16: uint16 bit patterns, scales None.
    """
    w13: np.ndarray
    w13_scales: np.ndarray | None
    w2: np.ndarray
    w2_scales: np.ndarray | None
    tensor_scales: np.ndarray


def gen_expert(cfg: LayerConfig, seed: int, layer: int, expert: int) -> ExpertWeights:
    H, F = cfg.hidden, cfg.ffn
    g = rng(seed, "expert", cfg.name, layer, expert)
    if cfg.wfmt == W_BF16:
        w13 = f32_to_bf16_bits(g.standard_normal((2 * F, H), dtype=np.float32) * np.float32(0.02))
        w2 = f32_to_bf16_bits(g.standard_normal((H, F), dtype=np.float32) * np.float32(0.02))
        return ExpertWeights(w13, None, w2, None, np.ones(2, np.float32))
    w13 = g.integers(0, 256, size=(2 * F, H // 2), dtype=np.uint8)
    w2 = g.integers(0, 256, size=(H, F // 2), dtype=np.uint8)
    if cfg.wfmt == W_MXFP4:
        # E8M0 codes 119..127 -> block scales 2^-8 .. 2^0
        s13 = g.integers(119, 128, size=(2 * F, H // 32), dtype=np.uint8)
        s2 = g.integers(119, 128, size=(H, F // 32), dtype=np.uint8)
        ts = np.ones(2, np.float32)
    else:
        # E4M3 codes 0x02..0x38 -> block scales 2^-8 .. 1.0 (subnormals included)
        s13 = g.integers(0x02, 0x39, size=(2 * F, H // 16), dtype=np.uint8)
        s2 = g.integers(0x02, 0x39, size=(H, F // 16), dtype=np.uint8)
        ts = g.uniform(0.5, 1.0, size=2).astype(np.float32)
    return ExpertWeights(w13, s13, w2, s2, ts)


def blob_alias(cfg: LayerConfig, layer: int, expert: int, distinct: int | None) -> tuple[int, int]:
    """(layer, expert) whose weights stand in for (layer, expert).

    With `distinct` set, only that many distinct expert weight sets exist and
    key l*E+e uses set (l*E+e) mod distinct.  Used where host RAM cannot hold
    every expert of a 40-layer model; cache semantics do not depend on it.
    """
    if not distinct:
        return layer, expert
    k = (layer * cfg.experts + expert) % distinct
    return k // cfg.experts, k % cfg.experts
