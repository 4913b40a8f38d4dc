"""Pins of the oracle's square-tile (2-D) block quantization against what does not depend on its
own code: the 1-D oracle on inputs where the two must agree, transposition consistency, a
hand-worked tile, and the half-step error bound."""
import numpy as np
import pytest

import oracle as O
from workloads import bf16_bits, bf16_to_f32

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float32)


def _tiles_with_equal_rows(R, C, bs, g):
    """Every bs x bs tile has bs identical rows (so each row segment's amax is the tile's)."""
    base = (g.standard_t(3, size=(R // bs, C)) * 0.3).astype(np.float32)
    base *= np.exp2(g.integers(-6, 7, size=(R // bs, 1))).astype(np.float32)
    return bf16_bits(np.repeat(base, bs, axis=0))


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("rnd", ["rtn", "sr"])
def test_equal_rows_reduce_to_1d_along_rows(fmt, rnd):
    bs = 32 if fmt == "mxfp4" else 16
    xb = _tiles_with_equal_rows(4 * bs, 6 * bs, bs, np.random.default_rng(1))
    r2 = O.quantize_2d(xb, fmt=fmt, rnd=rnd, seed=5)
    r1 = O.quantize(xb, fmt=fmt, axis=1, rnd=rnd, seed=5, tensor_scale=r2["tensor_scale"])
    np.testing.assert_array_equal(r2["scales"], r1["scales"])
    np.testing.assert_array_equal(r2["codes"], r1["codes"])


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("rnd", ["rtn", "sr"])
def test_equal_columns_reduce_to_1d_along_columns(fmt, rnd):
    bs = 32 if fmt == "mxfp4" else 16
    xt = _tiles_with_equal_rows(6 * bs, 4 * bs, bs, np.random.default_rng(2))
    xb = np.ascontiguousarray(xt.T)                      # tiles with identical columns
    r2 = O.quantize_2d(xb, fmt=fmt, rnd=rnd, seed=9)
    r1 = O.quantize(xb, fmt=fmt, axis=0, rnd=rnd, seed=9, tensor_scale=r2["tensor_scale"])
    np.testing.assert_array_equal(r2["scales_t"], r1["scales"])
    np.testing.assert_array_equal(r2["codes_t"], r1["codes"])


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_transposed_output_is_the_transpose(fmt):
    g = np.random.default_rng(3)
    bs = 32 if fmt == "mxfp4" else 16
    x = (g.standard_normal((3 * bs, 5 * bs)) * np.exp2(g.integers(-8, 8, size=(3 * bs, 1)))).astype(np.float32)
    r = O.quantize_2d(bf16_bits(x), fmt=fmt, rnd="sr", seed=11)
    d = O.dequantize(r["codes"], r["scales"], fmt=fmt, tensor_scale=r["tensor_scale"])
    dt = O.dequantize(r["codes_t"], r["scales_t"], fmt=fmt, tensor_scale=r["tensor_scale"])
    np.testing.assert_array_equal(dt, d.T)


def test_hand_worked_nv_tile():
    """16x16 NVFP4 tile of grid values with amax 6 and s_t = 2^-8: t = 6/6/2^-8 = 256 = E4M3 0x78,
    S = 256 * 2^-8 = 1, so every code is the grid index of its value with the sign bit."""
    i = np.arange(16)
    mag = GRID[(i[:, None] + i[None, :]) % 8]
    sign = np.where((i[:, None] * 3 + i[None, :]) % 5 == 0, -1.0, 1.0).astype(np.float32)
    x = mag * sign
    x[0, 0] = 6.0
    r = O.quantize_2d(bf16_bits(x), fmt="nvfp4", tensor_scale=np.float32(2.0 ** -8))
    assert np.all(r["scales"] == 0x78) and np.all(r["scales_t"] == 0x78)
    codes = np.searchsorted(GRID, np.abs(x)).astype(np.uint8) | np.where(np.signbit(x), 8, 0).astype(np.uint8)
    np.testing.assert_array_equal(r["codes"], O.pack_nibbles(codes))
    np.testing.assert_array_equal(r["codes_t"], O.pack_nibbles(np.ascontiguousarray(codes.T)))


def test_hand_worked_mx_tile():
    """32x32 MXFP4 tile with amax 6: E = floor(log2 6) - 2 = 0, byte 127, v = x."""
    i = np.arange(32)
    x = GRID[(i[:, None] * 5 + i[None, :]) % 8].astype(np.float32)
    x[3, 7] = 6.0
    r = O.quantize_2d(bf16_bits(x), fmt="mxfp4")
    assert np.all(r["scales"] == 127)
    codes = np.searchsorted(GRID, x).astype(np.uint8)
    np.testing.assert_array_equal(r["codes"], O.pack_nibbles(codes))


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_half_step_error_bound(fmt):
    g = np.random.default_rng(4)
    bs = 32 if fmt == "mxfp4" else 16
    x = bf16_to_f32(bf16_bits((g.standard_normal((8 * bs, 8 * bs)) * 0.7).astype(np.float32)))
    r = O.quantize_2d(bf16_bits(x), fmt=fmt)
    d = O.dequantize(r["codes"], r["scales"], fmt=fmt, tensor_scale=r["tensor_scale"]).astype(np.float64)
    if fmt == "mxfp4":
        S = np.ldexp(1.0, r["scales"].astype(np.int64) - 127)
    else:
        S = O.e4m3_decode(r["scales"]).astype(np.float64) * np.float64(r["tensor_scale"])
    S = np.repeat(S, bs, axis=1)
    v = np.abs(x) / S
    step = np.where(v < 2, 0.5, np.where(v < 4, 1.0, 2.0))
    inside = v <= 6
    slack = 0 if fmt == "mxfp4" else 2.0 ** -20 * 6 * S
    assert np.all(np.abs(x - d)[inside] <= (0.5 * step * S + slack)[inside])
