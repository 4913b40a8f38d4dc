"""Pins of the oracle's MSE-fitted grid scales (`oracle/mse_grid.py`): the MXFP4 clip-threshold
exponent against the OCP rule, the no-clipping bound and hand-worked block maxima; the fitted
threshold against the squared error it minimises; the NVFP4 search against errors computed from
the dequantized outputs (not from the oracle's own error routine), exact representability,
invariance under power-of-two scaling, and the exact integer objective against Python integers."""
import math

import ml_dtypes
import numpy as np
import pytest

import oracle as O
from oracle import mse_grid as M
from workloads import bf16_bits, bf16_to_f32, normal_bf16, student_t_bf16


def _all_positive_bf16():
    bits = np.arange(1, 0x7F80, dtype=np.uint16)              # every positive finite bf16 value
    return bf16_to_f32(bits)


def test_clip_8_is_the_ocp_rule():
    a = _all_positive_bf16()
    np.testing.assert_array_equal(M.mx_scale_exponent_clip(a, 8.0), O.mx_scale_exponent(a))
    assert M.mx_scale_exponent_clip(np.float32(0), 7.25) == -127


@pytest.mark.parametrize("T", [6.0, 7.25])
def test_block_max_lands_in_the_clip_window(T):
    """amax / 2^E lies in (T/2, T] whenever E is not clamped: the grid reaches amax (up to the
    clip) and the next smaller exponent would not."""
    a = _all_positive_bf16().astype(np.float64)
    E = M.mx_scale_exponent_clip(a, T)
    r = a / np.ldexp(1.0, E)
    free = (E > -127) & (E < 127)
    assert np.all(r[free] <= T) and np.all(r[free] > T / 2)


def test_hand_worked_block_maxima():
    # 7 = 1.75 * 2^2: 7 <= 7.25 * 2^0 -> E = 0 (OCP also 0); 7.5 > 7.25 -> E = 1 (OCP 0)
    assert M.mx_scale_exponent_clip(np.float32(7.0), 7.25) == 0
    assert M.mx_scale_exponent_clip(np.float32(7.25), 7.25) == 0
    assert M.mx_scale_exponent_clip(np.float32(7.5), 7.25) == 1
    assert O.mx_scale_exponent(np.float32(7.5)) == 0
    # 0.1 = 1.6 * 2^-4: 1.6 <= 7.25/4 -> E = -6
    assert M.mx_scale_exponent_clip(np.float32(0.1), 7.25) == -6
    # 0.115 = 1.84 * 2^-4: 1.84 > 1.8125 -> E = -5
    assert M.mx_scale_exponent_clip(np.float32(0.115), 7.25) == -5


def test_fitted_clip_threshold_minimises_rotated_gaussian_error():
    """On seeded Gaussian data rotated by 128-blocks of H/sqrt(128), the 1/16 grid of [6, 8] has its
    least MXFP4 RTN error at MX_GRID_CLIP, and the OCP threshold 8 costs over 4 % more."""
    g = np.random.default_rng([20, 7])
    x = O.block_hadamard(g.standard_normal((512, 4096)), 128).astype(np.float32)
    best, grid, errs = M.fit_mx_grid_clip(x)
    assert best == M.MX_GRID_CLIP
    assert errs[-1] > 1.04 * errs.min()


def test_mxfp4_gs_quantizer_uses_the_clip_threshold():
    x = np.zeros((1, 64), dtype=np.float32)
    x[0, 0] = 7.5                       # block 0: E = 1 under 7.25, E = 0 under OCP
    x[0, 32] = 7.0                      # block 1: E = 0 under both
    r = O.quantize(bf16_bits(x), fmt="mxfp4_gs")
    assert list(r["scales"][0]) == [128, 127]
    assert list(O.quantize(bf16_bits(x), fmt="mxfp4")["scales"][0]) == [127, 127]


# ------------------------------------------------------------------ NVFP4 ---

def _block_sse(xf, codes, scales, s_t):
    d = O.dequantize(codes, scales, fmt="nvfp4", tensor_scale=s_t).astype(np.float64)
    e = (xf.astype(np.float64) - d).reshape(xf.shape[0], -1, 16)
    return np.sum(e * e, axis=-1)


def _quantize_with(xf, scales, s_t):
    """RTN codes of xf under the given bytes and tensor scale, by the ordinary quantizer's arithmetic
    (each block's byte forced through its own tensor-scale-free path)."""
    S = (O.e4m3_decode(scales).astype(np.float32) * np.float32(s_t)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = (xf.reshape(xf.shape[0], -1, 16) / S[..., None]).astype(np.float32)
    c = np.where((scales == 0)[..., None], np.uint8(0), O.e2m1_rtn(v))
    return O.pack_nibbles(c.reshape(xf.shape))


@pytest.mark.parametrize("seed", [0, 1])
def test_block_step_never_worse_than_standard_or_four_over_six(seed):
    xb = student_t_bf16((32, 256), 3.0, 0.1, 30 + seed, 0)
    xf = bf16_to_f32(xb)
    r = O.quantize_mse(xb, iters=0)
    std = O.quantize(xb, fmt="nvfp4")
    f46 = O.quantize(xb, fmt="nvfp4_4o6")
    assert r["tensor_scale"] == std["tensor_scale"]
    e = _block_sse(xf, r["codes"], r["scales"], r["tensor_scale"])
    assert np.all(e <= _block_sse(xf, std["codes"], std["scales"], std["tensor_scale"]) * (1 + 1e-12))
    assert np.all(e <= _block_sse(xf, f46["codes"], f46["scales"], f46["tensor_scale"]) * (1 + 1e-12))
    assert e.sum() < 0.9 * _block_sse(xf, std["codes"], std["scales"], std["tensor_scale"]).sum()


def test_block_step_against_every_byte_of_the_window():
    """Brute force over the 17 window bytes with errors from the dequantized outputs: the chosen
    byte has the least error, and no earlier byte in the tie order has an equal one."""
    xb = normal_bf16((8, 128), 0.02, 31, 0)
    xf = bf16_to_f32(xb)
    s_t = O.nv_tensor_scale(xf)
    r = O.quantize_mse(xb, iters=0)
    t = ((np.max(np.abs(xf.reshape(8, -1, 16)), axis=-1) / np.float32(6)).astype(np.float32) / s_t).astype(np.float32)
    b6 = t.astype(ml_dtypes.float8_e4m3fn).view(np.uint8).astype(np.int64)
    order = [0] + [s * j for j in range(1, 9) for s in (-1, 1)]
    for i in range(8):
        for g in range(8):
            errs = []
            for off in order:
                b = np.uint8(min(max(b6[i, g] + off, 1), 126))
                sc = np.full((1, 1), b, dtype=np.uint8)
                blk = xf[i:i + 1, 16 * g:16 * g + 16]
                errs.append(float(_block_sse(blk, _quantize_with(blk, sc, s_t), sc, s_t)[0, 0]))
            k = int(np.argmin(errs))
            assert r["scales"][i, g] == np.uint8(min(max(b6[i, g] + order[k], 1), 126))


def test_block_exactly_on_another_grid_is_found():
    """Block 0 holds 0.65625 = 2688 * 2^-12, so s_t = 2^-12 exactly.  Block 1 holds G * 2^-6 with
    G up to 4: exact under the byte of 64 (S = 64 * 2^-12), while the standard byte is that of
    RN_E4M3(4 * 64 / 6) = 44, five bytes lower, whose grid leaves errors.  The search finds an
    exact byte: zero error."""
    vals = np.array([0, .5, 1, 1.5, 2, 3, 4, 4, -.5, -1, -2, -3, 1.5, .5, 3, -4], dtype=np.float32)
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, 0] = 0.65625
    x[0, 16:] = vals * np.float32(2.0 ** -6)
    xb = bf16_bits(x)
    r = O.quantize_mse(xb, iters=0)
    assert r["tensor_scale"] == np.float32(2.0 ** -12)
    xf = bf16_to_f32(xb)
    assert np.all(_block_sse(xf, r["codes"], r["scales"], r["tensor_scale"]) == 0.0)
    std = O.quantize(xb, fmt="nvfp4")
    assert std["scales"][0, 1] == np.float32(44.0).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert _block_sse(xf, std["codes"], std["scales"], std["tensor_scale"])[0, 1] > 0


def test_power_of_two_scaling_of_the_tensor_changes_only_s_t():
    """Scaling a tensor by 2 leaves s_t's multiplier alone and scales s_t by 2 (amax doubles), so
    every byte and code is unchanged: the search sees the same problem."""
    xb = student_t_bf16((16, 128), 3.0, 0.1, 32, 0)
    xf = bf16_to_f32(xb)
    r1 = O.quantize_mse(xb, iters=1)
    r2 = O.quantize_mse(bf16_bits(xf * np.float32(2)), iters=1)
    assert r2["tensor_scale"] == np.float32(2) * r1["tensor_scale"]
    np.testing.assert_array_equal(r1["scales"], r2["scales"])
    np.testing.assert_array_equal(r1["codes"], r2["codes"])


def test_exact_floor_sum_against_python_integers():
    g = np.random.default_rng(5)
    err = np.abs(g.standard_normal(5000)) * np.exp2(g.integers(-60, 6, size=5000))
    for P in (80, 90, 20):
        want = sum(int(math.floor(math.ldexp(float(v), P))) for v in err)
        assert M._exact_floor_sum(err, P) == want


def test_tensor_step_never_worse_than_keeping_the_scale():
    xb = normal_bf16((16, 256), 0.02, 33, 0)
    xf = bf16_to_f32(xb)
    x16 = xf.reshape(-1, 16)
    s0 = O.nv_tensor_scale(xf)
    P = M.objective_exponent(np.float32(np.max(np.abs(xf))))
    s1, sb1, Q = M.tensor_step(x16, s0, P)
    assert min(Q) == Q[8] or s1 != s0                        # k = 0 is candidate 8
    assert M.tensor_objective(x16, sb1, s1, P) == min(Q) <= Q[8]
    # the winner's error from the dequantized outputs is no larger than the start's (up to the
    # objective's truncation of < amax^2 2^-80 per block)
    codes1 = _quantize_with(xf, sb1.reshape(16, -1), s1)
    r0 = O.quantize_mse(xb, iters=0)
    e1 = _block_sse(xf, codes1, sb1.reshape(16, -1), s1).sum()
    e0 = _block_sse(xf, r0["codes"], r0["scales"], r0["tensor_scale"]).sum()
    assert e1 <= e0 + len(x16) * float(np.max(np.abs(xf))) ** 2 * 2.0 ** -80


def test_zero_tensor_and_iteration_bounds():
    r = O.quantize_mse(np.zeros((2, 32), dtype=np.uint16), iters=2)
    assert r["tensor_scale"] == 1.0 and not r["scales"].any() and not r["codes"].any()
    with pytest.raises(ValueError):
        O.quantize_mse(np.zeros((2, 32), dtype=np.uint16), iters=9)


def test_sr_uses_the_searched_scales():
    xb = student_t_bf16((8, 64), 3.0, 0.1, 34, 0)
    a = O.quantize_mse(xb, rnd="rtn", iters=1)
    b = O.quantize_mse(xb, rnd="sr", seed=7, iters=1)
    assert a["tensor_scale"] == b["tensor_scale"]
    np.testing.assert_array_equal(a["scales"], b["scales"])
    # SR codes are the RTN grid neighbours: dequantized values within one grid step of x
    xf = bf16_to_f32(xb)
    d = O.dequantize(b["codes"], b["scales"], fmt="nvfp4", tensor_scale=b["tensor_scale"])
    S = np.repeat(O.e4m3_decode(b["scales"]) * b["tensor_scale"], 16, axis=1)
    assert np.all(np.abs(d - xf) <= 2 * S + 1e-30)
