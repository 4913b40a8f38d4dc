"""Pins for the oracle's GEMM reference and scale-factor layout (CPU only)."""
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
from workloads import bf16_bits


def _q(x, fmt):
    return O.quantize(bf16_bits(np.asarray(x, np.float32)), fmt=fmt)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_gemm_brute_force_triple_loop(fmt):
    rng = np.random.default_rng(1)
    a = _q(rng.standard_normal((3, 64)), fmt)
    b = _q(rng.standard_normal((5, 64)) * 0.02, fmt)
    y, bound = O.gemm_ref(a, b, fmt)
    # brute force: decode every code and scale by hand, exact rational arithmetic
    bs = 32 if fmt == "mxfp4" else 16
    ca, cb = O.unpack_nibbles(a["codes"]), O.unpack_nibbles(b["codes"])

    def sc(byte):
        if fmt == "mxfp4":
            return Fraction(2) ** (int(byte) - 127)
        return Fraction(float(O.e4m3_decode(np.uint8(byte))))

    alpha = Fraction(1) if fmt == "mxfp4" else Fraction(float(a["tensor_scale"])) * Fraction(float(b["tensor_scale"]))
    for i in range(3):
        for j in range(5):
            acc = Fraction(0)
            tot = Fraction(0)
            for k in range(64):
                va = Fraction(float(O.e2m1_decode(ca[i, k]))) * sc(a["scales"][i, k // bs])
                vb = Fraction(float(O.e2m1_decode(cb[j, k]))) * sc(b["scales"][j, k // bs])
                acc += va * vb
                tot += abs(va * vb)
            assert abs(Fraction(y[i, j]) - alpha * acc) <= abs(alpha * acc) * Fraction(1, 2 ** 50)
            assert abs(Fraction(bound[i, j]) - abs(alpha) * tot) <= abs(alpha) * tot * Fraction(1, 2 ** 50)


def test_gemm_mx_small_is_exact():
    rng = np.random.default_rng(2)
    a = _q(rng.standard_normal((4, 128)), "mxfp4")
    b = _q(rng.standard_normal((4, 128)), "mxfp4")
    y, _ = O.gemm_ref(a, b, "mxfp4")
    da = O.deq_for_gemm(a["codes"], a["scales"], "mxfp4")
    db = O.deq_for_gemm(b["codes"], b["scales"], "mxfp4")
    for i in range(4):
        for j in range(4):
            exact = sum(Fraction(float(p)) * Fraction(float(q)) for p, q in zip(da[i], db[j]))
            assert Fraction(y[i, j]) == exact


def test_gemm_one_hot_weights_select_columns():
    rng = np.random.default_rng(3)
    a = _q(rng.standard_normal((8, 64)), "mxfp4")
    w = np.zeros((64, 64), np.float32)
    w[np.arange(64), np.arange(64)] = 4.0          # one-hot rows: block max 4 -> E = 0, code 6 (value 4)
    b = _q(w, "mxfp4")
    y, _ = O.gemm_ref(a, b, "mxfp4")
    np.testing.assert_array_equal(y, 4.0 * O.deq_for_gemm(a["codes"], a["scales"], "mxfp4"))


def test_gemm_sampled_rows_cols_match_full():
    rng = np.random.default_rng(4)
    a = _q(rng.standard_normal((40, 96)), "nvfp4")
    b = _q(rng.standard_normal((24, 96)), "nvfp4")
    y, bd = O.gemm_ref(a, b, "nvfp4")
    rows = np.array([0, 7, 39])
    yr, br = O.gemm_ref_rows(a, b, "nvfp4", rows)
    np.testing.assert_array_equal(yr, y[rows])
    cols = np.array([1, 23])
    yc, bc = O.gemm_ref_cols(a, b, "nvfp4", cols)
    np.testing.assert_array_equal(yc, y[:, cols])
    assert np.all(np.abs(y) <= bd)


def test_sf_layout_hand_positions_and_roundtrip():
    s = np.zeros((130, 9), np.uint8)
    s[33, 1] = 7          # tile (0,0): (33 % 32) * 16 + (33 // 32) * 4 + 1 = 21
    s[128, 0] = 9         # tile (1,0): start (1 * 3 + 0) * 512 = 1536
    s[5, 6] = 11          # tile (0,1): 512 + 5*16 + 0*4 + 2 = 594
    flat = O.sf_to_mma(s)
    assert flat.size == 256 * 12
    assert flat[21] == 7 and flat[1536] == 9 and flat[594] == 11
    rng = np.random.default_rng(0)
    s = rng.integers(1, 255, (300, 13), dtype=np.uint8)
    flat = O.sf_to_mma(s)
    np.testing.assert_array_equal(O.sf_from_mma(flat, 300, 13), s)
    assert np.count_nonzero(flat) == s.size            # pads are zero, no collisions
