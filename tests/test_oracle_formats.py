"""Pins for the oracle's number formats and dequantisation (CPU only).

E2M1 against the OCP MX table (golden fixture); E8M0 and E4M3 against
torch's own float8 decoders over all 256 codes; the canonical packed
layout (even column in the low nibble, one scale per 32 or 16 columns of a
row) against hand-worked blocks.
"""
import math
import os

import numpy as np
import pytest
import torch

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _read_e2m1():
    tab = {}
    for line in open(os.path.join(GOLD, "e2m1_table.txt")):
        if line.strip() and not line.startswith("#"):
            c, v = line.split()
            tab[int(c)] = float(v)
    return tab


def test_e2m1_table(orc):
    tab = _read_e2m1()
    assert len(tab) == 16
    for c, v in tab.items():
        got = orc.e2m1(c)
        assert got == v and math.copysign(1, got) == math.copysign(1, v), (c, got, v)


def test_e8m0_all_codes_match_torch(orc):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).double().numpy()
    for c in range(256):
        got = orc.e8m0(c)
        if math.isnan(ref[c]):
            assert math.isnan(got) and c == 255
        else:
            assert got == ref[c], c


def test_e4m3_all_codes_match_torch(orc):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    nans = 0
    for c in range(256):
        got = orc.e4m3(c)
        if math.isnan(ref[c]):
            assert math.isnan(got)
            nans += 1
        else:
            assert got == ref[c] and math.copysign(1, got) == math.copysign(1, ref[c]), c
    assert nans == 2  # S.1111.111 only


def _worked():
    rows = []
    for line in open(os.path.join(GOLD, "worked_blocks.txt")):
        if line.startswith(("mxfp4", "nvfp4")):
            head, vals = line.split("->")
            rows.append((head.split(), [float(v) for v in vals.split()]))
    return rows


def _pack_row(codes):
    """Pack codes of one row, even column -> low nibble (the documented layout)."""
    codes = np.asarray(codes, np.uint8)
    return (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)


def test_worked_mxfp4_blocks(orc):
    codes = np.arange(64) % 16
    q = _pack_row(codes)[None, :]
    sc = np.array([[126, 129]], np.uint8)
    got = orc.dequant_matrix(1, q, sc, 1.0, 1, 64)[0]
    w = [v for h, v in _worked() if h[0] == "mxfp4"]
    np.testing.assert_array_equal(got, np.array(w[0] + w[1]))


def test_worked_nvfp4_blocks(orc):
    codes = np.arange(32) % 16
    q = _pack_row(codes)[None, :]
    sc = np.array([[0x3C, 0x03]], np.uint8)
    got = orc.dequant_matrix(2, q, sc, np.float32(0.75), 1, 32)[0]
    w = [v for h, v in _worked() if h[0] == "nvfp4"]
    np.testing.assert_array_equal(got, np.array(w[0] + w[1]))


@pytest.mark.parametrize("wfmt,block", [(1, 32), (2, 16)])
def test_dequant_layout_two_rows(orc, wfmt, block):
    """Row stride and per-row scale indexing: row 1 must not read row 0's data."""
    rng = np.random.default_rng(3)
    cols = 4 * block
    codes = rng.integers(0, 16, size=(2, cols))
    q = np.stack([_pack_row(codes[0]), _pack_row(codes[1])])
    if wfmt == 1:
        sc = rng.integers(120, 130, size=(2, cols // block)).astype(np.uint8)
        scale = lambda c: 2.0 ** (int(c) - 127)
    else:
        sc = rng.integers(0x08, 0x40, size=(2, cols // block)).astype(np.uint8)
        ref = torch.tensor(sc.reshape(-1)).view(torch.float8_e4m3fn).double().numpy().reshape(sc.shape)
        scale = None
    ts = np.float32(0.625)
    got = orc.dequant_matrix(wfmt, q, sc, ts, 2, cols)
    e2 = _read_e2m1()
    for r in range(2):
        for c in range(cols):
            s = scale(sc[r, c // block]) if wfmt == 1 else ref[r, c // block] * float(ts)
            assert got[r, c] == e2[int(codes[r, c])] * s


def test_bf16_widening(orc):
    x = np.array([1.0, -2.5, 3.140625, 1e-3], np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    got = orc.dequant_matrix(0, bits, None, 1.0, 1, 4)[0]
    ref = torch.tensor(x).to(torch.bfloat16).double().numpy()
    # the first three are exact in bf16 (truncation == rounding there)
    np.testing.assert_array_equal(got[:3], ref[:3])
