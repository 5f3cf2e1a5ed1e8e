"""Pins for the oracle's scalar formats (E2M1, E4M3, Codebook10).

Each check ties the oracle to something other than itself: the page-printed
Codebook10 levels, PyTorch's float8_e4m3fn decoder and cast, or exact rational
brute force over the grid.
"""
import os
import random
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#")[0].strip()
        if line:
            k, *v = line.split()
            out[k] = v
    return out


def f32(v: float) -> float:
    return struct.unpack("<f", struct.pack("<f", v))[0]


def f32_next(v: float, d: int) -> float:
    """Neighbouring binary32 value (d = +1 / -1) of a non-negative float."""
    b = struct.unpack("<I", struct.pack("<f", v))[0]
    return struct.unpack("<f", struct.pack("<I", b + d))[0]


def brute_nearest(v: Fraction, grid):
    """Index of the nearest grid value, ties to the even index, saturating (exact)."""
    a = abs(v)
    if a >= grid[-1]:
        return len(grid) - 1
    best = min(range(len(grid)), key=lambda i: (abs(a - grid[i]), i % 2))
    return best


# ---------------------------------------------------------------- E2M1 -----
def test_e2m1_magnitudes_are_codebook10_halved_before_retune():
    """rocmwhy 01: Codebook10 is E2M1-derived with the outer 12 retuned to 10, so
    2*E2M1 magnitudes must be the Codebook10 levels with 10 replaced by 12."""
    g = _golden("rocmwhy_lab.txt")
    cb = [int(v) for v in g["codebook10"]]
    outer = int(g["e2m1_derived_outer"][0])
    expect = cb[:-1] + [outer]
    got = [2 * O.e2m1_decode(c) for c in range(8)]
    assert got == expect
    # the maximum magnitude 6 is the divisor of the NVFP4 block-scale recipe
    assert max(got) / 2 == 6


def test_e2m1_sign_bit():
    for c in range(8):
        assert O.e2m1_decode(c | 8) == -O.e2m1_decode(c)
    assert np.signbit(O.e2m1_decode(8))  # 0x8 decodes to -0 (numerically zero)


def test_e2m1_encode_matches_exact_nearest():
    grid = [Fraction(O.e2m1_decode(i)) for i in range(8)]
    vals = set()
    for i in range(7):
        mid = float((grid[i] + grid[i + 1]) / 2)
        for v in (mid, f32_next(mid, 1), f32_next(mid, -1)):
            vals.add(v)
    for q in grid:
        vals.add(float(q))
    rnd = random.Random(7)
    for _ in range(3000):
        vals.add(f32(rnd.uniform(0, 8)))
        vals.add(f32(10 ** rnd.uniform(-8, 2)))
    vals |= {0.0, 6.0, 7.0, f32_next(7.0, 1), 1e30, float("inf")}
    for v in vals:
        for s in (1, -1):
            x = s * v
            c = O.e2m1_encode(x)
            idx = brute_nearest(Fraction(v) if np.isfinite(v) else Fraction(10 ** 40), grid)
            assert c & 7 == idx, (x, c, idx)
            assert (c >> 3) == (1 if s < 0 else 0), (x, c)


def test_e2m1_ties_go_to_even():
    # 0.25 between 0 and 0.5 -> 0; 0.75 between 0.5 and 1 -> 1 (index 2); 5 -> 4 (index 6)
    assert O.e2m1_encode(0.25) == 0
    assert O.e2m1_encode(0.75) == 2
    assert O.e2m1_encode(1.25) == 2
    assert O.e2m1_encode(1.75) == 4
    assert O.e2m1_encode(2.5) == 4
    assert O.e2m1_encode(3.5) == 6
    assert O.e2m1_encode(5.0) == 6
    assert O.e2m1_encode(-0.0) == 8
    assert O.e2m1_encode(-0.2) == 8


# ---------------------------------------------------------------- E4M3 -----
def test_e4m3_decode_matches_torch_float8_e4m3fn():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([O.e4m3_decode(b) for b in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    m = ~np.isnan(ref)
    assert np.array_equal(got[m], ref[m])


def test_e4m3_facts_from_pages():
    # 6 * 448 in the global-scale recipe: 448 is the largest finite E4M3 value.
    assert O.e4m3_decode(0x7E) == 448.0
    assert all(O.e4m3_decode(b) < 448.0 for b in range(0x7E))
    # rocmwhy 02 readout 0.813 / 0.094: both are UE4M3 values shown to 3 decimals
    g = _golden("rocmwhy_lab.txt")
    finite = [O.e4m3_decode(b) for b in range(0x7F)]
    for shown in g["half_scales_shown"]:
        assert any(abs(v - float(shown)) < 5e-4 for v in finite), shown
    # 127 finite non-negative candidates ("full finite UE4M3 candidate set")
    assert len(set(finite)) == 127 and np.all(np.diff(finite) > 0)


def _e4m3_test_values():
    grid = [O.e4m3_decode(i) for i in range(127)]
    vals = set()
    for i in range(126):
        mid = f32((grid[i] + grid[i + 1]) / 2)
        vals |= {mid, f32_next(mid, 1), f32_next(mid, -1) if mid > 0 else mid}
        vals.add(grid[i])
    rnd = random.Random(11)
    for _ in range(20000):
        vals.add(f32(2.0 ** rnd.uniform(-14, 8.85)))
    vals |= {0.0, 2.0 ** -10, 2.0 ** -11, 1e-30, 447.9, 448.0}
    return sorted(v for v in vals if v < 464.0)


def test_e4m3_encode_matches_torch_cast_in_range():
    vals = _e4m3_test_values()
    ref = torch.tensor(vals, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([O.e4m3_encode(v) for v in vals], dtype=np.uint8)
    bad = np.nonzero(ref != got)[0]
    assert bad.size == 0, [(vals[i], got[i], ref[i]) for i in bad[:5]]
    neg = torch.tensor(vals[::37], dtype=torch.float32).neg().to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(neg, [O.e4m3_encode(-v) for v in vals[::37]])


def test_e4m3_saturates_above_448():
    for v in (448.0, 463.9, 464.0, 500.0, 1e38, float("inf")):
        assert O.e4m3_encode(v) == 0x7E
        assert O.e4m3_encode(-v) == 0xFE
    assert O.e4m3_encode(float("nan")) == 0x7F


def test_e4m3_lab_seed_rounds_to_shown_half_scale():
    # rocmwhy 02/03: search seeded near max_abs/10.  A half whose outlier is 8.2
    # seeds at 0.82, whose nearest UE4M3 value 0.8125 is the shown 0.813.
    assert O.e4m3_decode(O.e4m3_encode(f32(0.82))) == 0.8125


# ---------------------------------------------------------- Codebook10 -----
def test_codebook10_levels_match_page():
    cb = [int(v) for v in _golden("rocmwhy_lab.txt")["codebook10"]]
    assert [O.cb10_decode(c) for c in range(8)] == cb
    assert [O.cb10_decode(c | 8) for c in range(1, 8)] == [-v for v in cb[1:]]


def test_codebook10_snap_lab_readout():
    """rocmwhy 01 explorer readout: probe snaps to 3.0 with absolute error 0.30."""
    g = _golden("rocmwhy_lab.txt")
    for probe in g["snap_probe_values"]:
        idx = O.cb10_index(float(probe), 1.0)
        level = O.cb10_decode(idx)
        assert level == float(g["snap_result"][0])
        assert abs(abs(float(probe) - level) - float(g["snap_abs_error"][0])) < 1e-6


@pytest.mark.parametrize("s_code", [0x01, 0x07, 0x08, 0x1C, 0x35, 0x38, 0x50, 0x7E])
def test_codebook10_index_is_exact_nearest(s_code):
    s = O.e4m3_decode(s_code)
    grid = [Fraction(s) * v for v in (0, 1, 2, 3, 4, 6, 8, 10)]
    rnd = random.Random(s_code)
    vals = set()
    for i in range(7):
        mid = float((grid[i] + grid[i + 1]) / 2)
        vals |= {mid, f32_next(mid, 1), f32_next(mid, -1)}
    for _ in range(500):
        vals.add(f32(rnd.uniform(0, 12 * s)))
    for v in vals:
        assert O.cb10_index(v, s) == brute_nearest(Fraction(v), grid), (v, s)
