"""Pins of the oracle's activation-term encoding (orc_act_terms): the FP4
tensor-core path writes every activation row as a short sum of E2M1 terms
with block scales of the weights' scale type.

Pinned by hand-worked blocks (tests/golden/act_terms_blocks.txt) and by
properties the definition fixes: each scale is the smallest of its format
that covers the block's remaining magnitude; each code is the nearest E2M1
value (checked against the golden E2M1 table, ties to the even code); the
terms of T are the first terms of T+1; negating a row negates its codes;
blocks that are E2M1 values times a scale are exact after one term; the
reconstruction error shrinks geometrically with T; the NVFP4 row exponent
puts the row's largest magnitude in [2^10, 2^11).
"""
import os

import numpy as np
import pytest
import torch

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _e2m1_table():
    vals = {}
    for line in open(os.path.join(GOLD, "e2m1_table.txt")):
        line = line.split("#")[0].split()
        if len(line) >= 2:
            vals[int(line[0])] = float(line[1])
    return np.array([vals[c] for c in range(16)])


E2M1 = _e2m1_table()


def _scale_values(wfmt):
    """Scale code -> value, decoded by torch (independent of the oracle)."""
    codes = torch.arange(256, dtype=torch.uint8)
    if wfmt == 1:
        return codes.view(torch.float8_e8m0fnu).double().numpy()
    return codes.view(torch.float8_e4m3fn).double().numpy()


def _golden():
    blocks = {}
    for line in open(os.path.join(GOLD, "act_terms_blocks.txt")):
        line = line.split("#")[0].split()
        if not line:
            continue
        b = blocks.setdefault(line[0], {})
        if "=" in line[1]:
            b.update({k: int(v) for k, v in (t.split("=") for t in line[1:])})
        else:
            b[line[1]] = [float(v) for v in line[2:]]
    return blocks


def _recon(codes, scales, p, wfmt):
    """x ~ 2^-p sum_t e2m1(codes_t) * scale(scales_t), float64."""
    sv = _scale_values(wfmt)
    T, K = codes.shape
    vs = K // scales.shape[1]
    tot = np.zeros(K)
    for t in range(T):
        tot += E2M1[codes[t]] * np.repeat(sv[scales[t]], vs)
    return tot * 2.0 ** -p


@pytest.mark.parametrize("name", ["A", "B"])
def test_hand_worked_blocks(orc, name):
    g = _golden()[name]
    x = np.zeros((1, g["K"]), np.float32)
    x[0, :len(g["x"])] = g["x"]
    codes, scales, p = orc.act_terms(x, g["wfmt"], g["T"])
    assert p[0] == g["p"]
    assert list(scales[0, :, 0]) == [int(v) for v in g["scales"]]
    for t in range(g["T"]):
        want = [int(v) for v in g[f"codes{t}"]]
        assert list(codes[0, t, :len(want)]) == want
        assert not codes[0, t, len(want):].any()


def _rows(seed, n, K):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, K)).astype(np.float32)
    x[1] *= 1e-6                                   # tiny row
    x[2] = np.float32(1e5) * rng.standard_normal(K).astype(np.float32)   # large row
    x[3, ::3] = 0.0                                # zeros inside blocks
    x[4] = np.round(x[4] * 4) / 4                  # many exact ties on the grids
    return x


@pytest.mark.parametrize("wfmt", [1, 2])
def test_scales_minimal_and_codes_nearest(orc, wfmt):
    K, T = 256, 4
    vs = 32 if wfmt == 1 else 16
    x = _rows(1, 6, K)
    codes, scales, p = orc.act_terms(x, wfmt, T)
    sv = _scale_values(wfmt)
    ok_codes = np.arange(1, 255) if wfmt == 1 else np.arange(1, 0x7F)
    for i in range(x.shape[0]):
        r = x[i].astype(np.float64) * 2.0 ** p[i]
        for t in range(T):
            s = np.repeat(sv[scales[i, t]], vs)
            m = np.abs(r).reshape(-1, vs).max(1)
            for b in range(K // vs):
                if m[b] == 0:
                    continue
                sb = sv[scales[i, t, b]]
                below = sv[ok_codes][sv[ok_codes] < sb]
                # covers the block (the fp32 rounding of the residual is far below 1e-6)
                assert 6 * sb >= m[b] * (1 - 1e-6), (i, t, b)
                if below.size:
                    assert 6 * below.max() < m[b] * (1 + 1e-6), (i, t, b)
            # nearest E2M1 of r / s, ties to the even code
            a = r / s
            dist = np.abs(a[:, None] - E2M1[None, :8] * np.sign(a)[:, None])
            q = codes[i, t]
            d_q = np.abs(a - E2M1[q])
            assert np.all(d_q <= dist.min(1) + 1e-9 * np.abs(a)), (i, t)
            if wfmt == 1 and t == 0:
                # first MXFP4 term: r / s is exact here, so exact ties go to the even code
                tie = np.sum(dist == dist.min(1, keepdims=True), axis=1) > 1
                assert tie.sum() > 0 or i != 4
                assert np.all((q[tie] & 1) == 0), (i, q[tie])
            r = r - E2M1[q] * s


@pytest.mark.parametrize("wfmt", [1, 2])
def test_prefix_sign_exact_and_convergence(orc, wfmt):
    K = 512
    x = _rows(2, 6, K)
    c3, s3, p3 = orc.act_terms(x, wfmt, 3)
    c5, s5, p5 = orc.act_terms(x, wfmt, 5)
    np.testing.assert_array_equal(c3, c5[:, :3])
    np.testing.assert_array_equal(s3, s5[:, :3])
    np.testing.assert_array_equal(p3, p5)
    cn, sn, pn = orc.act_terms(-x, wfmt, 3)
    np.testing.assert_array_equal(sn, s3)
    np.testing.assert_array_equal(cn, np.where(c3 > 0, c3 ^ 8, 0))
    errs = []
    for T in (1, 2, 3, 4, 5):
        c, s, p = orc.act_terms(x, wfmt, T)
        e = max(np.linalg.norm(_recon(c[i], s[i], p[i], wfmt) - x[i]) / np.linalg.norm(x[i])
                for i in range(x.shape[0]))
        errs.append(e)
    assert errs[0] < 0.2
    for a, b in zip(errs, errs[1:]):
        assert b < a / 4, errs
    assert errs[2] < 4e-3 and errs[3] < 6e-4


@pytest.mark.parametrize("wfmt", [1, 2])
def test_exact_blocks_and_zero_row(orc, wfmt):
    vs = 32 if wfmt == 1 else 16
    rng = np.random.default_rng(3)
    q = rng.integers(0, 16, size=(2, 64))
    x = (E2M1[q] * 0.25).astype(np.float32)     # E2M1 values times a power of two
    x[:, ::vs] = 6 * 0.25                       # every block reaches 6 * scale
    c, s, p = orc.act_terms(x, wfmt, 3)
    np.testing.assert_allclose(_recon(c[0], s[0], p[0], wfmt), x[0], rtol=0, atol=0)
    assert not c[:, 1:].any()
    z = np.zeros((1, 64), np.float32)
    c, s, p = orc.act_terms(z, wfmt, 2)
    assert not c.any() and p[0] == 0
    assert np.all(s == (127 if wfmt == 1 else 0x38))


def test_nvfp4_row_exponent(orc):
    x = _rows(4, 6, 128)
    _, _, p = orc.act_terms(x, 2, 1)
    mx = np.abs(x).max(1).astype(np.float64) * 2.0 ** p
    assert np.all((mx >= 1024) & (mx < 2048)), (p, mx)
    _, _, p1 = orc.act_terms(x, 1, 1)
    assert not p1.any()
