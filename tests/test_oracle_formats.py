"""Pins of the oracle's element formats against what the pages and the
format definitions fix (no GPU).

* E2M1 magnitudes: "What is NVFP4? 4-bit AI inference on NVIDIA Blackwell
  explained", "What does NVFP4 mean?" (tests/golden/e2m1_magnitudes.txt).
* Encoders: brute-force nearest-value search written here (not the oracle's
  arithmetic) over a dense sweep of binary32 inputs, ties to the even code,
  saturation at the largest finite value.
* E4M3 (the block-scale type named in "NVFP4 Explained", "Why the Block Scale
  Uses FP8 E4M3"): closed-form facts of the OCP FP8 E4M3 definition -- 127
  finite non-negative codes, maximum 448, smallest subnormal 2^-9, smallest
  normal 2^-6, 3 mantissa bits.
"""
import os

import numpy as np
import pytest

import oracle as O


def _golden_mags(golden_dir):
    vals = []
    with open(os.path.join(golden_dir, "e2m1_magnitudes.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                vals.append(float(line))
    return vals


def test_e2m1_magnitudes_round_trip(golden_dir):
    mags = _golden_mags(golden_dir)
    assert mags == sorted(mags) and len(mags) == 8
    # codes 0..7 are the magnitudes in increasing order, 8..15 their negatives
    decoded = [O.e2m1_decode(c) for c in range(16)]
    assert decoded[:8] == mags
    assert decoded[8:] == [-m for m in mags]
    for m in mags:
        for v in (m, -m):
            assert O.e2m1_decode(O.e2m1_encode(v)) == v
    assert max(mags) == 6.0


def _sweep_f32(max_pattern, extra_points):
    """Dense binary32 sweep: every 256th bit pattern below max_pattern, the same
    patterns with a pseudo-random low byte, and +-8 ulps around extra_points."""
    base = np.arange(0, max_pattern, 256, dtype=np.uint64)
    low = (base * np.uint64(2654435761)) >> np.uint64(8)
    jitter = base | (low & np.uint64(0xFF))
    pats = np.concatenate([base, jitter]).astype(np.uint32)
    vals = pats.view(np.float32)
    pts = []
    for p in extra_points:
        c = np.array([p], np.float32).view(np.uint32)[0]
        for d in range(-8, 9):
            q = np.int64(c) + d
            if q >= 0:
                pts.append(np.uint32(q))
    vals = np.concatenate([vals, np.array(pts, np.uint32).view(np.float32)])
    return vals[np.isfinite(vals)]


def _nearest_with_even_ties(a, table):
    """Index of the nearest entry of the ascending table; ties go to the even
    index; values beyond the last entry take the last entry."""
    a = a.astype(np.float64)
    hi = np.clip(np.searchsorted(table, a), 1, len(table) - 1)
    lo = hi - 1
    dlo = np.abs(a - table[lo])
    dhi = np.abs(table[hi] - a)
    pick = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo % 2 == 0, lo, hi)))
    pick = np.where(a >= table[-1], len(table) - 1, pick)
    pick = np.where(a <= table[0], 0, pick)
    return pick


def test_e2m1_encode_matches_bruteforce(golden_dir):
    table = np.array(_golden_mags(golden_dir), np.float64)
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 1e-30, 0.5, 1.0]
    pos = _sweep_f32(0x41800000, mids)           # magnitudes below 16
    vals = np.concatenate([pos, -pos, np.array([1e30, -1e30, 7.0, -6.5], np.float32)])
    got = O.e2m1_encode_array(vals)
    want = _nearest_with_even_ties(np.abs(vals), table).astype(np.uint8)
    want |= (np.signbit(vals).astype(np.uint8) << 3)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first {vals[bad[:5]]} got {got[bad[:5]]} want {want[bad[:5]]}"


def test_e2m1_tie_cases_and_sign_of_zero():
    # ties go to the even code (mantissa bit 0)
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for v, want in ties.items():
        assert O.e2m1_decode(O.e2m1_encode(v)) == want
        assert O.e2m1_decode(O.e2m1_encode(-v)) == -want
    assert O.e2m1_encode(-0.0) == 0x8 and O.e2m1_encode(0.0) == 0x0
    assert O.e2m1_encode(-0.1) == 0x8
    assert O.e2m1_encode(100.0) == 0x7 and O.e2m1_encode(-100.0) == 0xF


def _e4m3_table():
    return np.array([O.e4m3_decode(c) for c in range(0x7F)], np.float64)


def test_e4m3_closed_form_facts():
    t = _e4m3_table()
    assert t[0] == 0.0
    assert np.all(np.diff(t) > 0), "codes 0x00..0x7E must increase strictly"
    assert t[0x7E] == 448.0                      # largest finite E4M3
    assert t[0x01] == 2.0 ** -9                  # smallest subnormal
    assert t[0x08] == 2.0 ** -6                  # smallest normal
    assert np.all(np.mod(t * 512.0, 1.0) == 0.0)  # every value is a multiple of 2^-9
    # 3 mantissa bits: inside each binade [2^e, 2^(e+1)) there are 8 equally spaced values
    for e in range(-6, 9):
        b = t[(t >= 2.0 ** e) & (t < 2.0 ** (e + 1))]
        assert len(b) == (7 if e == 8 else 8)
        assert np.allclose(np.diff(b), 2.0 ** (e - 3), rtol=0, atol=0)
    assert np.isnan(O.e4m3_decode(0x7F)) or O.e4m3_decode(0x7F) == 480.0  # never produced


def test_e4m3_round_trip():
    for c in range(0x7F):
        assert O.e4m3_encode(O.e4m3_decode(c)) == c


def test_e4m3_encode_matches_bruteforce():
    t = _e4m3_table()
    mids = list((t[1:] + t[:-1]) / 2.0) + [448.0, 464.0, 480.0, 2.0 ** -10, 1e-45]
    vals = _sweep_f32(0x44800000, mids)          # [0, 1024)
    vals = vals[vals >= 0]
    got = O.e4m3_encode_array(vals)
    want = _nearest_with_even_ties(vals, t).astype(np.uint8)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first {vals[bad[:5]]} got {got[bad[:5]]} want {want[bad[:5]]}"
    # saturation: everything at or above the top of the range maps to 448
    assert O.e4m3_encode(1e30) == 0x7E and O.e4m3_encode(448.0) == 0x7E
