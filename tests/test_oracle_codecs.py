"""Pins for the oracle's element and scale codecs (CPU only).

Each check compares the oracle with something other than itself: the code
points printed on "Hardware FP4 inference for speech on Blackwell" (section
"NVFP4, and the two ways it fails"), its E4M3 maximum of 448, and
independent nearest-value searches (numpy here, C in tests/native/sweep.c)
over every positive finite binary32 value.
"""
import ctypes

import numpy as np
import pytest

from tests.golden import load as golden


def test_e2m1_decode_matches_printed_code_points(orc):
    pts = golden.e2m1_codepoints()
    assert [orc.e2m1_decode(c) for c in range(8)] == pts
    assert [orc.e2m1_decode(8 + c) for c in range(8)] == [-p for p in pts]
    assert np.signbit(orc.e2m1_decode(8))            # code 0x8 is -0


def _brute_e2m1(v: np.ndarray, pts) -> np.ndarray:
    """Nearest printed code point, ties to the even code, |v| > 6 -> 6."""
    pts = np.asarray(pts)
    a = np.abs(v)[:, None]
    d = np.abs(a - pts[None, :])
    best = d.min(axis=1, keepdims=True)
    tie_ok = (d == best)
    # among the tied candidates prefer an even code index
    even = (np.arange(8) % 2 == 0)[None, :]
    pick = np.where((tie_ok & even).any(axis=1), np.argmax(tie_ok & even, axis=1),
                    np.argmax(tie_ok, axis=1))
    pick = np.where(np.abs(v) >= pts[-1], 7, pick)      # saturate above 6
    return pick.astype(np.uint8) | np.where(np.signbit(v), 8, 0).astype(np.uint8)


def test_e2m1_encode_vs_numpy_brute_force(orc):
    pts = golden.e2m1_codepoints()
    g = np.random.default_rng(123)
    mids = [(pts[i] + pts[i + 1]) / 2 for i in range(7)]
    special = []
    for m in mids + pts:
        special += [m, np.nextafter(m, 0), np.nextafter(m, 10)]
    v = np.concatenate([g.uniform(-8, 8, 200000), np.array(special),
                        -np.array(special), [0.0, -0.0, 6.0, 7.0, 1e30, -1e30]])
    got = orc.e2m1_encode_array(v)
    want = _brute_e2m1(v, pts)
    assert np.array_equal(got, want)


def test_e2m1_tie_rule_and_sign(orc):
    # ties go to the even code: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4
    for v, m in [(0.25, 0), (0.75, 1), (1.25, 1), (1.75, 2), (2.5, 2), (3.5, 4), (5.0, 4),
                 (6.5, 6), (100.0, 6)]:
        c = orc.e2m1_encode(v)
        assert orc.e2m1_decode(c) == m
        assert orc.e2m1_encode(-v) == c | 8
    assert orc.e2m1_encode(-0.1) == 0x8                  # negative -> -0
    assert orc.e2m1_encode(-0.0) == 0x8


@pytest.mark.slow
def test_e2m1_exhaustive_sweep(sweep_lib):
    fb = ctypes.c_uint32(0)
    bad = sweep_lib.sweep_e2m1(1, 0x7F800000, ctypes.byref(fb))
    assert bad == 0, f"first mismatch at bits {fb.value:#010x}"


def test_e4m3_grid_facts(orc):
    facts = golden.format_facts()
    vals = [orc.e4m3_decode(c) for c in range(0x7F)]
    assert max(vals) == facts["e4m3_max"] == orc.e4m3_decode(0x7E)
    assert np.isnan(orc.e4m3_decode(0x7F))
    assert all(b > a for a, b in zip(vals, vals[1:]))    # strictly increasing
    assert orc.e4m3_decode(1) == 2.0 ** -9                # smallest subnormal
    assert orc.e4m3_decode(0x08) == 2.0 ** -6             # smallest normal
    # E4M3 has 3 mantissa bits: 160 and 176 are neighbours near 166.7
    assert orc.e4m3_decode(orc.e4m3_encode(166.67)) == 160.0


def test_e4m3_saturates_at_448(orc):
    facts = golden.format_facts()
    for v in [448.0, 450.0, 463.9, 464.0, 480.0, 603.0, 1e30]:
        assert orc.e4m3_decode(orc.e4m3_encode(v)) == facts["e4m3_max"]


def test_e4m3_encode_vs_numpy_brute_force(orc):
    grid = np.array([orc.e4m3_decode(c) for c in range(0x7F)])
    g = np.random.default_rng(7)
    v = np.concatenate([np.exp(g.uniform(np.log(1e-4), np.log(600), 200000)),
                        (grid[1:] + grid[:-1]) / 2, grid]).astype(np.float32)
    got = orc.e4m3_encode_array(v)
    a = v.astype(np.float64)[:, None]
    d = np.abs(a - grid[None, :])
    best = d.min(axis=1, keepdims=True)
    tie = d == best
    even = (np.arange(0x7F) % 2 == 0)[None, :]
    want = np.where((tie & even).any(axis=1), np.argmax(tie & even, axis=1),
                    np.argmax(tie, axis=1))
    want = np.where(v >= 448, 0x7E, want)
    assert np.array_equal(got, want.astype(np.uint8))


@pytest.mark.slow
def test_e4m3_exhaustive_sweep(sweep_lib):
    fb = ctypes.c_uint32(0)
    bad = sweep_lib.sweep_e4m3(1, 0x7F800000, ctypes.byref(fb))
    assert bad == 0, f"first mismatch at bits {fb.value:#010x}"


def test_e8m0_is_power_of_two(orc):
    assert orc.e8m0_decode(127) == 1.0
    assert orc.e8m0_decode(0) == 2.0 ** -127
    assert orc.e8m0_decode(254) == 2.0 ** 127
    assert np.isnan(orc.e8m0_decode(255))
