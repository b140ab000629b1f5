"""Pins for the oracle's permutation, SwiGLU experts and combine (CPU only).

Permutation against numpy's stable argsort; the expert FFN against numpy
matrix products plus the closed-form silu; the whole tiny layer against
hand-computed values (golden fixture); x = 0, identical experts and k = 1
as special cases.
"""
import math
import os

import numpy as np
import pytest

from expert_cached_sparse_b200 import workloads as W

GOLD = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("n,e,k", [(1, 8, 2), (37, 16, 3), (300, 256, 6), (5, 4, 4)])
def test_permute_is_stable_argsort(orc, n, e, k):
    rng = np.random.default_rng(n)
    idx = rng.integers(0, e, size=(n, k)).astype(np.int32)
    offsets, row_of, assign_of = orc.permute(idx, e)
    flat = idx.reshape(-1)
    ref_assign = np.argsort(flat, kind="stable")
    np.testing.assert_array_equal(assign_of, ref_assign)
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=e))]))
    np.testing.assert_array_equal(row_of[assign_of], np.arange(n * k))


def test_permute_empty(orc):
    offsets, row_of, assign_of = orc.permute(np.zeros((0, 2), np.int32), 5)
    assert list(offsets) == [0] * 6 and row_of.size == 0


@pytest.mark.parametrize("h,f", [(8, 1), (16, 24), (64, 32)])
def test_ffn_matches_numpy(orc, h, f):
    rng = np.random.default_rng(h * f)
    w13 = rng.standard_normal((2 * f, h))
    w2 = rng.standard_normal((h, f))
    x = rng.standard_normal(h)
    g = w13[:f] @ x
    u = w13[f:] @ x
    hv = g / (1.0 + np.exp(-g)) * u
    ref = w2 @ hv
    np.testing.assert_allclose(orc.expert_ffn(w13, w2, x), ref, rtol=1e-12, atol=1e-12)


def test_ffn_zero_input(orc):
    rng = np.random.default_rng(0)
    w13 = rng.standard_normal((8, 16))
    w2 = rng.standard_normal((16, 4))
    y = orc.expert_ffn(w13, w2, np.zeros(16))
    assert np.all(y == 0.0)


def _golden_tiny():
    vals = {}
    for line in open(os.path.join(GOLD, "tiny_layer.txt")):
        if line.strip() and not line.startswith("#"):
            tok = line.split()
            vals[tok[0]] = [float(t) for t in tok[1:]]
    return vals


def _tiny_weights():
    H = 8
    e0 = np.zeros((2, H)); e0[0, 0] = 1; e0[1, 1] = 1
    e1 = np.zeros((2, H)); e1[0, 1] = 1; e1[1, 0] = 1
    w2_0 = np.array([1, -1, 0.5, 0, 0, 0, 0, 0], np.float64)[:, None]
    w2_1 = np.array([0, 0, 1, 2, 0, 0, 0, 0], np.float64)[:, None]
    bits = lambda a: W.f32_to_bf16_bits(np.asarray(a, np.float32))
    ex = [W.ExpertWeights(bits(e0), None, bits(w2_0), None, np.ones(2, np.float32)),
          W.ExpertWeights(bits(e1), None, bits(w2_1), None, np.ones(2, np.float32))]
    wg = np.zeros((2, H), np.float32); wg[0, 0] = 1; wg[1, 1] = 1
    x = np.array([[1, 2, 0, 0, 0, 0, 0, 0]], np.float32)
    return x, bits(wg), ex


@pytest.mark.parametrize("k", [1, 2])
def test_tiny_layer_hand_values(orc, k):
    gold = _golden_tiny()
    x, wg, ex = _tiny_weights()
    out, idx, w, logits = orc.moe_layer(x, wg, None, k, W.W_BF16, 8, 1, lambda e: ex[e])
    assert list(idx[0]) == [int(v) for v in gold[f"k{k}_idx"]]
    np.testing.assert_allclose(w[0], gold[f"k{k}_w"], rtol=1e-15)
    np.testing.assert_allclose(out[0], gold[f"k{k}_out"], rtol=1e-14, atol=1e-15)
    assert math.isclose(gold["h0"][0], 2 / (1 + math.exp(-1)))


def test_identical_experts_give_ffn_regardless_of_routing(orc):
    cfg = W.scaled(W.TINY, hidden=64, ffn=32, experts=6, top_k=3)
    rng = np.random.default_rng(9)
    ew = W.gen_expert(cfg, 0, 0, 0)
    x = rng.standard_normal((7, 64)).astype(np.float32)
    wg = W.gen_wg(cfg, 0, 0)
    out, idx, w, _ = orc.moe_layer(x, wg, None, 3, W.W_BF16, 64, 32, lambda e: ew)
    w13, w2 = orc.dequant_expert(W.W_BF16, ew, 64, 32)
    for t in range(7):
        np.testing.assert_allclose(out[t], orc.expert_ffn(w13, w2, x[t].astype(np.float64)),
                                   rtol=1e-12, atol=1e-9)


def test_combine_weights_linear(orc):
    rng = np.random.default_rng(4)
    y = rng.standard_normal((6, 5))
    w = rng.random((2, 3))
    out = orc.combine(y, w)
    ref = np.stack([w[t] @ y[3 * t:3 * t + 3] for t in range(2)])
    np.testing.assert_allclose(out, ref, rtol=1e-14)


def test_token_subset_equals_full(orc):
    cfg = W.scaled(W.DS_DECODE, hidden=256, ffn=64, experts=8, top_k=2)
    x = W.gen_x(cfg, 0, 12)
    wg = W.gen_wg(cfg, 0, 0)
    b = W.gen_bias(cfg, 0, 0)
    fn = lambda e: W.gen_expert(cfg, 0, 0, e)
    full = orc.moe_layer(x, wg, b, 2, cfg.wfmt, 256, 64, fn)[0]
    sub = orc.moe_layer(x, wg, b, 2, cfg.wfmt, 256, 64, fn, tokens=[3, 7, 11])[0]
    np.testing.assert_array_equal(sub, full[[3, 7, 11]])
