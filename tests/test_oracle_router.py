"""Pins for the oracle's router (CPU only).

Logits: exact integer dot products where fp32 is exact, and an fp64 numpy
dot within the fp32 rounding bound elsewhere.  Selection: brute-force sort
by (-logit, index).  Weights: torch softmax over all experts, renormalised
over the selected set; k = E is the plain softmax, k = 1 gives 1.0.
"""
import numpy as np
import pytest
import torch

from expert_cached_sparse_b200 import workloads as W


def _bits(a):
    return W.f32_to_bf16_bits(np.asarray(a, np.float32))


def test_integer_logits_exact(orc):
    rng = np.random.default_rng(0)
    n, h, e = 5, 512, 12
    x = rng.integers(-8, 9, size=(n, h)).astype(np.float32)
    wg = rng.integers(-8, 9, size=(e, h)).astype(np.float32)
    bias = rng.integers(-100, 100, size=e).astype(np.float32)
    logits, idx, w = orc.router(x, _bits(wg), bias, 3)
    ref = x.astype(np.int64) @ wg.astype(np.int64).T + bias.astype(np.int64)
    np.testing.assert_array_equal(logits, ref.astype(np.float32))


@pytest.mark.parametrize("h", [8, 256, 264, 4096])
def test_logits_within_fp32_bound(orc, h):
    rng = np.random.default_rng(h)
    n, e = 4, 16
    x = rng.standard_normal((n, h)).astype(np.float32)
    wgb = _bits(rng.standard_normal((e, h)) * 0.02)
    wg = W.bf16_bits_to_f32(wgb).astype(np.float64)
    bias = rng.standard_normal(e).astype(np.float32)
    logits, _, _ = orc.router(x, wgb, bias, 2)
    ref = x.astype(np.float64) @ wg.T + bias
    mag = np.abs(x.astype(np.float64)) @ np.abs(wg).T + np.abs(bias)
    bound = (h + 8) * 2.0 ** -24 * mag
    assert np.all(np.abs(logits - ref) <= bound)


def test_topk_is_bruteforce_sort(orc):
    rng = np.random.default_rng(1)
    n, h, e, k = 32, 256, 64, 6
    x = W.f32_to_bf16_bits(rng.standard_normal((n, h)))
    wgb = _bits(rng.standard_normal((e, h)) * 0.02)
    # duplicate some gate rows so exact ties occur
    wgb[5] = wgb[9]
    wgb[40] = wgb[2]
    logits, idx, _ = orc.router(x, wgb, None, k)
    for t in range(n):
        order = sorted(range(e), key=lambda j: (-float(logits[t, j]), j))
        assert list(idx[t]) == order[:k]
        if 9 in idx[t] and 5 in idx[t]:
            assert list(idx[t]).index(5) < list(idx[t]).index(9)


@pytest.mark.parametrize("k", [1, 3, 8, 64])
def test_weights_are_renormalised_softmax(orc, k):
    rng = np.random.default_rng(k)
    n, h, e = 16, 128, 64
    x = rng.standard_normal((n, h)).astype(np.float32)
    wgb = _bits(rng.standard_normal((e, h)) * 0.3)
    bias = (rng.standard_normal(e) * 2).astype(np.float32)
    logits, idx, w = orc.router(x, wgb, bias, k)
    p = torch.softmax(torch.tensor(logits, dtype=torch.float64), dim=-1).numpy()
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    ref = sel / sel.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(w, ref, rtol=1e-12, atol=1e-15)
    if k == 1:
        assert np.all(w == 1.0)
    if k == e:
        np.testing.assert_allclose(np.take_along_axis(w, np.argsort(idx, axis=1), axis=1), p,
                                   rtol=1e-12, atol=1e-15)
    # descending logit order
    lsel = np.take_along_axis(logits, idx.astype(np.int64), axis=1)
    assert np.all(np.diff(lsel, axis=1) <= 0)


def test_nan_logits_rank_last(orc):
    h, e, k = 16, 5, 3
    x = np.ones((2, h), np.float32)
    x[0, 3] = np.nan
    wg = np.zeros((e, h), np.float32)
    wg[:, 0] = [1, 2, 3, 4, 5]
    logits, idx, _ = orc.router(x, _bits(wg), None, k)
    assert np.all(np.isnan(logits[0]))
    assert list(idx[0]) == [0, 1, 2]          # all NaN: ties -> lower index
    assert list(idx[1]) == [4, 3, 2]


def test_hand_example(orc):
    """H=8, E=3: logits (1, 2, 2): tie between 1 and 2 goes to expert 1."""
    x = np.array([[1, 2, 0, 0, 0, 0, 0, 0]], np.float32)
    wg = np.zeros((3, 8), np.float32)
    wg[0, 0] = 1
    wg[1, 1] = 1
    wg[2, 0] = 2
    logits, idx, w = orc.router(x, _bits(wg), None, 2)
    assert list(logits[0]) == [1.0, 2.0, 2.0]
    assert list(idx[0]) == [1, 2]
    assert list(w[0]) == [0.5, 0.5]
