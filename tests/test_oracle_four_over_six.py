"""Pins of the oracle's four-over-six NVFP4 block scaling against hand-worked blocks, the E4M3
library cast, and an error invariant computed from the dequantized outputs (not from the
oracle's own error routine)."""
import ml_dtypes
import numpy as np
import pytest

import oracle as O
from workloads import bf16_bits, bf16_to_f32

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float32)


def _e4m3_byte(v):
    return int(np.array(v, dtype=np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8))


def test_block_exact_on_the_four_grid_takes_four():
    """x = k * (grid values up to 4), k = 2^-4, s_t = 2^-8: t4 = 0.25/4/2^-8 = 16 (exact in E4M3)
    makes every element exact (err4 = 0), while t6 = 10.67 rounds to 11 and leaves errors."""
    k = np.float32(2.0 ** -4)
    vals = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 4, -0.5, -1, -2, -3, 1.5, 0.5, 3, -4], dtype=np.float32)
    x = (vals * k)[None, :]
    r = O.quantize(bf16_bits(x), fmt="nvfp4_4o6", tensor_scale=np.float32(2.0 ** -8))
    assert r["scales"][0, 0] == _e4m3_byte(16.0)
    codes = np.searchsorted(GRID, np.abs(vals)).astype(np.uint8) | np.where(np.signbit(vals), 8, 0).astype(np.uint8)
    np.testing.assert_array_equal(r["codes"], O.pack_nibbles(codes[None, :]))
    r6 = O.quantize(bf16_bits(x), fmt="nvfp4", tensor_scale=np.float32(2.0 ** -8))
    assert r6["scales"][0, 0] == _e4m3_byte(11.0)


def test_block_exact_on_the_six_grid_keeps_six():
    k = np.float32(2.0 ** -4)
    vals = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -6, -4, 3, 2, 1, 0.5, -1.5, 6], dtype=np.float32)
    x = (vals * k)[None, :]
    st = np.float32(2.0 ** -8)
    r = O.quantize(bf16_bits(x), fmt="nvfp4_4o6", tensor_scale=st)
    r6 = O.quantize(bf16_bits(x), fmt="nvfp4", tensor_scale=st)
    np.testing.assert_array_equal(r["scales"], r6["scales"])
    np.testing.assert_array_equal(r["codes"], r6["codes"])


def _block_sse(xf, codes, scales, s_t):
    d = O.dequantize(codes, scales, fmt="nvfp4", tensor_scale=s_t).astype(np.float64)
    e = (xf.astype(np.float64) - d).reshape(xf.shape[0], -1, 16)
    return np.sum(e * e, axis=-1)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_never_worse_than_six_and_picks_four_somewhere(seed):
    g = np.random.default_rng(seed)
    x = (g.standard_t(4, size=(64, 256)) * np.exp2(g.integers(-5, 5, size=(64, 1)))).astype(np.float32)
    xb = bf16_bits(x)
    xf = bf16_to_f32(xb)
    r = O.quantize(xb, fmt="nvfp4_4o6")
    r6 = O.quantize(xb, fmt="nvfp4")
    assert r["tensor_scale"] == r6["tensor_scale"]
    sse46 = _block_sse(xf, r["codes"], r["scales"], r["tensor_scale"])
    sse6 = _block_sse(xf, r6["codes"], r6["scales"], r6["tensor_scale"])
    assert np.all(sse46 <= sse6 * (1 + 1e-12))
    changed = r["scales"] != r6["scales"]
    assert 0.05 < changed.mean() < 0.95
    # blocks that took the four-scale never use the code for 6
    c = O.unpack_nibbles(r["codes"]).reshape(64, -1, 16)
    assert not np.any((c[changed] & 7) == 7)


def test_saturated_candidates_fall_back_to_six():
    """Blocks at the tensor's amax: t6 = 448 and t4 = 672 both saturate to 448, so the block keeps
    the standard scale and codes."""
    g = np.random.default_rng(5)
    x = (g.standard_normal((4, 64)) * 0.1).astype(np.float32)
    x[:, ::16] = 3.0                                    # every block holds the tensor's amax
    xb = bf16_bits(x)
    r = O.quantize(xb, fmt="nvfp4_4o6")
    r6 = O.quantize(xb, fmt="nvfp4")
    assert np.all(r6["scales"] == _e4m3_byte(448.0))
    np.testing.assert_array_equal(r["scales"], r6["scales"])
    np.testing.assert_array_equal(r["codes"], r6["codes"])


def test_axis0_and_sr_use_the_same_choice():
    """The choice depends on the block's values only: along axis 0 it matches axis 1 on the
    transpose, and SR keeps RTN's choice of scale."""
    g = np.random.default_rng(6)
    xb = bf16_bits(g.standard_normal((48, 32)).astype(np.float32))
    st = np.float32(0.01)
    a0 = O.quantize(xb, fmt="nvfp4_4o6", axis=0, tensor_scale=st)
    a1 = O.quantize(np.ascontiguousarray(xb.T), fmt="nvfp4_4o6", axis=1, tensor_scale=st)
    np.testing.assert_array_equal(a0["scales"], a1["scales"])
    np.testing.assert_array_equal(a0["codes"], a1["codes"])
    sr = O.quantize(xb, fmt="nvfp4_4o6", rnd="sr", seed=3, tensor_scale=st)
    rt = O.quantize(xb, fmt="nvfp4_4o6", tensor_scale=st)
    np.testing.assert_array_equal(sr["scales"], rt["scales"])
