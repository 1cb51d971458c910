"""Pins for the oracle's E2M1 / E4M3 codecs (CPU only).

E2M1 follows the 1-2-1 bit split of "Serving sub-second Ideogram v4 without quality
loss", section "Running the transformer in FP4"; E4M3 is the block-scale format.
The pins are hand-written golden tables, torch's own float8_e4m3fn conversion (a
library routine), and the nearest-level property checked on dense grids.
"""
import os

import numpy as np
import pytest
import torch

from oracle import nvfp4_oracle as o

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                a, b = line.split()
                rows.append((float(a), float(b)))
    return rows


def test_e2m1_decode_all_16_codes_golden():
    tab = _table("e2m1_levels.txt")
    assert len(tab) == 16
    codes = np.array([int(c) for c, _ in tab])
    want = np.array([v for _, v in tab])
    got = o.e2m1_decode(codes)
    assert np.array_equal(got, want)
    # the sign bit of the negative zero code is kept
    assert np.signbit(got[8]) and not np.signbit(got[0])


def test_e2m1_encode_ties_and_saturation_golden():
    for x, code in _table("e2m1_rne_ties.txt"):
        assert int(o.e2m1_encode(np.float32(x))) == int(code), x


def test_e2m1_encode_is_nearest_with_even_ties_on_dense_grid():
    x = np.linspace(-8, 8, 200001).astype(np.float32)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    x = np.concatenate([x, mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 9)])
    c = o.e2m1_encode(x)
    v = o.e2m1_decode(c)
    levels = o.e2m1_decode(np.arange(16))
    best = np.min(np.abs(x.astype(np.float64)[:, None] - levels[None, :]), axis=1)
    err = np.abs(v - x.astype(np.float64))
    assert np.all(err <= best + 0.0)
    # at exact ties the chosen code has mantissa bit 0 (unless saturated)
    tie = np.isin(np.abs(x), mids)
    assert np.all((c[tie] & 1) == 0)
    # sign follows the input
    nz = v != 0
    assert np.all(np.sign(v[nz]) == np.sign(x[nz]))


def test_e2m1_roundtrip_levels():
    codes = np.arange(16, dtype=np.uint8)
    vals = o.e2m1_decode(codes).astype(np.float32)
    back = o.e2m1_encode(vals)
    # every code reproduces itself, including 0x8 (negative zero)
    assert np.array_equal(back, codes)


def test_e4m3_decode_all_256_codes_against_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = o.e4m3_decode(codes)
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.all(both_nan | (ref == got))
    assert np.sum(np.isnan(got)) == 2   # 0x7F and 0xFF


def test_e4m3_golden_points():
    for code, val in _table("e4m3_points.txt"):
        assert o.e4m3_decode(int(code)) == val
        assert int(o.e4m3_encode(np.float32(val))) == int(code)


def test_e4m3_encode_matches_torch_rne_in_range():
    grid = np.linspace(0, 448, 400001).astype(np.float32)
    vals = o.e4m3_decode(np.arange(0x7F))
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    x = np.concatenate([grid, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
                        np.float32([2.0 ** -10, 2.0 ** -11, 1e-30])])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(o.e4m3_encode(x), ref)


def test_e4m3_saturates_at_448():
    x = np.float32([448.0, 449.0, 463.9, 464.0, 480.0, 1e6, 3e38])
    assert np.all(o.e4m3_encode(x) == 0x7E)
    with pytest.raises(ValueError):
        o.e4m3_encode(np.float32([-1.0]))
