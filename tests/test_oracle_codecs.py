"""Pins of the oracle's E2M1 / UE4M3 codecs against the pages' printed grid
and against an independent library (ml_dtypes' float4_e2m1fn and
float8_e4m3fn, both round-to-nearest-even)."""
import ml_dtypes
import numpy as np
import pytest

import oracle as O
from conftest import golden_dict, read_golden


def test_e2m1_grid_matches_printed_grid():
    grid = [float(v) for v in read_golden("e2m1_grid.txt")[0]]
    assert len(grid) == 8
    for c in range(8):
        assert O.e2m1_value(c) == grid[c]
        assert O.e2m1_value(c | 8) == -grid[c]
    assert max(abs(O.e2m1_value(c)) for c in range(16)) == golden_dict("format_constants.txt")["e2m1_max"]


def test_e2m1_decode_matches_library():
    lib_vals = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    for c in range(16):
        assert O.e2m1_value(c) == lib_vals[c]


def test_e2m1_encode_roundtrip_every_code():
    for c in range(16):
        if c == 8:                       # -0 is canonicalised to +0
            assert O.e2m1_encode(O.e2m1_value(c)) == 0
            continue
        assert O.e2m1_encode(O.e2m1_value(c)) == c


def test_e2m1_encode_matches_library_sweep():
    # dense sweep over [-8, 8] including every midpoint between grid values
    xs = np.concatenate([np.linspace(-8, 8, 20001, dtype=np.float32),
                         np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32),
                         -np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32),
                         np.array([1e-30, -1e-30, 100.0, -100.0, 6.0001], np.float32)])
    ref = xs.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 15
    ref = np.where(ref == 8, 0, ref)     # library keeps -0; the oracle writes +0
    got = np.array([O.e2m1_encode(float(x)) for x in xs])
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, list(zip(xs[bad][:5], got[bad][:5], ref[bad][:5]))


def test_e2m1_midpoints_round_half_even():
    # (midpoint, expected magnitude) read off the grid: ties go to the even code
    table = [(0.25, 0.0), (0.75, 1.0), (1.25, 1.0), (1.75, 2.0), (2.5, 2.0), (3.5, 4.0), (5.0, 4.0)]
    for x, want in table:
        assert O.e2m1_value(O.e2m1_encode(x)) == want
        assert O.e2m1_value(O.e2m1_encode(-x)) == -want or want == 0.0


def test_ue4m3_decode_matches_library():
    lib_vals = np.arange(128, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for c in range(127):
        assert O.ue4m3_value(c) == lib_vals[c]
    assert np.isnan(O.ue4m3_value(0x7F))
    assert O.ue4m3_value(0x7E) == golden_dict("format_constants.txt")["e4m3_max"]


def test_ue4m3_encode_matches_library_sweep():
    rng = np.random.default_rng(5)
    xs = np.concatenate([
        np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448.0), 40000)).astype(np.float32),
        np.array([O.ue4m3_value(c) for c in range(1, 127)], np.float32),
        # exact midpoints between neighbouring codes
        np.array([(O.ue4m3_value(c) + O.ue4m3_value(c + 1)) / 2 for c in range(0, 126)], np.float32),
    ])
    ref = xs.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    got = np.array([O.ue4m3_encode(float(x)) for x in xs])
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, list(zip(xs[bad][:5], got[bad][:5], ref[bad][:5]))


@pytest.mark.parametrize("x", [448.0, 449.0, 463.9, 464.0, 1000.0, 1e30])
def test_ue4m3_saturates_at_448(x):
    assert O.ue4m3_encode(x) == 0x7E


def test_ue4m3_zero_and_subnormal_ties():
    assert O.ue4m3_encode(0.0) == 0
    assert O.ue4m3_encode(2.0 ** -10) == 0          # half of the smallest subnormal: tie to even (0)
    assert O.ue4m3_encode(1.5 * 2.0 ** -9) == 2     # tie between codes 1 and 2 -> 2
    assert O.ue4m3_encode(2.0 ** -9) == 1


def test_global_scale_rule():
    # Eq. 5: gamma * amax / 6 = 448 for the tensor's largest block
    for amax in [6.0, 1.0, 0.0625, 3.14159]:
        g = O.global_scale(amax)
        assert abs(g * amax / 6 - 448.0) <= 448.0 * 2 ** -22
    assert O.global_scale(0.0) == 1.0
