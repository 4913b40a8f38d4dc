"""Pins for the oracle's element/scale formats (CPU only).

Library cross-checks (ml_dtypes casts are called, not copied) and closed forms.
"""
import os

import ml_dtypes
import numpy as np
import pytest

from oracle import formats as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_e2m1():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "e2m1_values.txt")) if l[0] != "#" and l.strip()]
    return {int(c): float(v) for c, v in rows}


def test_e2m1_decode_matches_published_table():
    table = _golden_e2m1()
    got = F.e2m1_decode(np.arange(16))
    for c in range(16):
        assert got[c] == table[c]
        assert np.signbit(got[c]) == np.signbit(table[c])


def test_e2m1_decode_matches_ml_dtypes():
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(F.e2m1_decode(np.arange(16)), lib)


def _sweep_fp32():
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    mids = np.array([.25, .75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0], np.float32)
    pts = np.concatenate([grid, mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(9)),
                          np.linspace(0, 8, 200001, dtype=np.float32),
                          np.float32(2.0) ** np.arange(-149, -60, dtype=np.float32),
                          np.array([1e30, 3.0e38], np.float32)])
    return np.concatenate([pts, -pts]).astype(np.float32)


def test_e2m1_rtn_matches_ml_dtypes_cast():
    v = _sweep_fp32()
    lib = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    np.testing.assert_array_equal(F.e2m1_rtn(v), lib)


def test_e2m1_rtn_closed_form_ties():
    # ties go to the even code: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4; >6 saturates
    v = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 100.0, -0.1, -0.0], np.float32)
    want = [0, 2, 2, 4, 4, 6, 6, 7, 7, 8, 8]
    np.testing.assert_array_equal(F.e2m1_rtn(v), want)


def test_e4m3_decode_matches_ml_dtypes():
    b = np.arange(256, dtype=np.uint8)
    lib = b.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    got = F.e4m3_decode(b)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(lib))
    ok = ~np.isnan(lib)
    np.testing.assert_array_equal(got[ok], lib[ok])
    assert F.e4m3_decode(np.uint8(0x7E)) == 448.0


def test_e4m3_rne_matches_ml_dtypes_below_max():
    vals = F.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    t = np.concatenate([vals.astype(np.float32), mids, np.nextafter(mids, np.float32(0)),
                        np.nextafter(mids, np.float32(1e9)),
                        np.linspace(0, 448, 100001, dtype=np.float32),
                        np.float32(2.0) ** np.arange(-20, 9, 0.125, dtype=np.float32)]).astype(np.float32)
    t = t[t <= 448]
    lib = t.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    np.testing.assert_array_equal(F.e4m3_rne_sat(t), lib)


def test_e4m3_saturates_above_max():
    # ml_dtypes returns NaN above 448; the reading clamps to 448 (byte 0x7E) first
    np.testing.assert_array_equal(F.e4m3_rne_sat(np.array([449, 464, 500, 1e6], np.float32)), [0x7E] * 4)


def test_mx_scale_exponent_closed_form():
    rng = np.random.default_rng(7)
    amax = np.abs(rng.standard_normal(100000).astype(np.float32)) * np.float32(2.0) ** rng.integers(-100, 100, 100000).astype(np.float32)
    amax = amax[amax > 0].astype(np.float32)
    E = F.mx_scale_exponent(amax)
    inside = (E > -127) & (E < 127)
    # 4 * 2^E <= amax < 8 * 2^E : the block max lands in [4, 8)
    lo = np.ldexp(4.0, E)
    hi = np.ldexp(8.0, E)
    assert np.all((lo <= amax)[inside]) and np.all((amax < hi)[inside])
    # library cross-check on normal values: floor(log2)
    np.testing.assert_array_equal(E[inside], np.floor(np.log2(amax.astype(np.float64)))[inside].astype(np.int64) - 2)


def test_mx_scale_exponent_boundaries():
    for k in range(-120, 120, 7):
        p = np.float32(2.0) ** np.float32(k)
        below = np.nextafter(p, np.float32(0))
        above = np.nextafter(p, np.float32(np.inf))
        assert F.mx_scale_exponent(p) == k - 2
        assert F.mx_scale_exponent(below) == k - 3
        assert F.mx_scale_exponent(above) == k - 2
    assert F.mx_scale_exponent(np.float32(0)) == -127
    assert F.mx_scale_exponent(np.float32(2.0 ** -130)) == -127      # clamped (fp32 subnormal)
    assert F.mx_scale_exponent(np.float32(3.0e38)) == 125


@pytest.mark.parametrize("p", [0.1, 0.25, 0.5, 0.9])
def test_sr_unbiased_every_interval(p):
    grid = [0, .5, 1, 1.5, 2, 3, 4, 6]
    n = 100000
    rng = np.random.default_rng(11)
    for lo, hi in zip(grid[:-1], grid[1:]):
        x = np.float32(lo + p * (hi - lo))
        r = rng.integers(0, 2 ** 32, n, dtype=np.uint64).astype(np.uint32)
        for sgn in (1, -1):
            codes = F.e2m1_sr(np.full(n, sgn * x, np.float32), r)
            vals = F.e2m1_decode(codes)
            assert set(np.unique(np.abs(vals))) <= {lo, hi}
            pe = (float(x) - lo) / (hi - lo)
            tol = 5 * (hi - lo) * np.sqrt(pe * (1 - pe) / n)
            assert abs(vals.mean() - sgn * float(x)) <= tol


def test_sr_grid_points_and_saturation():
    r = np.array([0, 1, 2 ** 31, 2 ** 32 - 1], np.uint64)
    for g, c in zip([0, .5, 1, 1.5, 2, 3, 4, 6], range(8)):
        np.testing.assert_array_equal(F.e2m1_sr(np.full(4, g, np.float32), r), [c] * 4)
    np.testing.assert_array_equal(F.e2m1_sr(np.full(4, 7.5, np.float32), r), [7] * 4)
    np.testing.assert_array_equal(F.e2m1_sr(np.full(4, -100.0, np.float32), r), [15] * 4)


def test_sr_threshold_exact():
    # x = 0.75 -> p = 0.5 exactly -> threshold 2^31: r = 2^31 - 1 rounds up, r = 2^31 stays down
    x = np.full(2, 0.75, np.float32)
    np.testing.assert_array_equal(F.e2m1_sr(x, np.array([2 ** 31 - 1, 2 ** 31], np.uint64)), [2, 1])
