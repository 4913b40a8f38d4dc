"""Pins for the oracle's MXFP4/NVFP4 quantizer (CPU only).

Closed forms worked by hand from the format definitions, invariants
(idempotence, the half-grid-step error bound, SR unbiasedness at the tensor
level), special cases (zero blocks, saturation, subnormal scales) and
reductions (axis 0 == axis 1 of the transpose).
"""
import ml_dtypes
import numpy as np
import pytest

import oracle as O
from workloads import bf16_bits, bf16_to_f32


def q(x32, **kw):
    return O.quantize(bf16_bits(np.asarray(x32, np.float32)), **kw)


def codes_of(res):
    return O.unpack_nibbles(res["codes"])


# --- hand-worked blocks --------------------------------------------------------

def test_mx_worked_block_unit_scale():
    # amax 6 -> floor(log2 6) = 2 -> E = 0 -> byte 127, v = x; ties go to the even code
    x = np.zeros((1, 32), np.float32)
    x[0, :12] = [6, 5, 3.5, 2.5, 1.75, 1.25, 0.75, 0.25, -6, -5, -0.1, 0]
    r = q(x, fmt="mxfp4")
    assert r["scales"].tolist() == [[127]]
    assert codes_of(r)[0, :12].tolist() == [7, 6, 6, 4, 4, 2, 2, 0, 15, 14, 8, 0]


def test_mx_worked_block_saturation_and_small_scale():
    # amax 7 -> E = 0, 7 saturates to 6 (code 7)
    x = np.zeros((1, 64), np.float32)
    x[0, 0] = 7.0
    # second block: amax 0.75 -> floor(log2 .75) = -1 -> E = -3 (byte 124): 0.75*8 = 6 -> code 7;
    # bf16(0.1) = 0.10009765625, *8 = 0.80078125 -> nearest 1.0 -> code 2
    x[0, 32] = 0.75
    x[0, 33] = 0.1
    r = q(x, fmt="mxfp4")
    assert r["scales"].tolist() == [[127, 124]]
    c = codes_of(r)[0]
    assert c[0] == 7 and c[32] == 7 and c[33] == 2


def test_mx_packing_nibble_order():
    x = np.zeros((1, 32), np.float32)
    x[0, 0], x[0, 1] = 1.0, 6.0            # amax 6 -> E = 0: codes 2 and 7
    r = q(x, fmt="mxfp4")
    assert r["codes"][0, 0] == (2 | (7 << 4))


def test_nv_worked_blocks():
    # tensor amax 2688 -> s_t = 1 exactly
    x = np.zeros((1, 48), np.float32)
    x[0, 0] = 2688.0                       # block 0: t = 448 -> byte 0x7E, S = 448, v = 6 -> code 7
    x[0, 16] = 6.0                         # block 1: t = 1 -> byte 0x38 (1.0), v = x
    x[0, 17] = 2.5                         #   tie 2/3 -> code 4 (2.0)
    x[0, 32] = 0.001                       # block 2: t = 1.67e-4 < 2^-10 -> sb = 0 -> all codes +0
    r = q(x, fmt="nvfp4")
    assert r["tensor_scale"] == np.float32(1.0)
    assert r["scales"].tolist() == [[0x7E, 0x38, 0x00]]
    c = codes_of(r)[0]
    assert c[0] == 7 and c[16] == 7 and c[17] == 4 and c[32] == 0


def test_nv_tensor_scale_closed_form():
    x = np.zeros((2, 16), np.float32)
    x[1, 3] = -3.0
    r = q(x, fmt="nvfp4")
    assert r["tensor_scale"] == np.float32(np.float32(3.0) / np.float32(2688.0))
    assert q(np.zeros((2, 16)), fmt="nvfp4")["tensor_scale"] == np.float32(1.0)


def test_zero_blocks_are_positive_zero():
    x = np.zeros((2, 64), np.float32)
    x[0, :32] = -0.0
    for fmt in ("mxfp4", "nvfp4"):
        r = q(x, fmt=fmt)
        assert np.all(codes_of(r) == 0)
        assert np.all(r["scales"] == 0)


# --- invariants ------------------------------------------------------------------

def _deq(r, fmt):
    return O.dequantize(r["codes"], r["scales"], fmt=fmt, tensor_scale=r["tensor_scale"])


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_idempotent_on_grid(fmt):
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((64, 256)) * np.exp(rng.standard_normal((64, 1)))).astype(np.float32)
    bs = 32 if fmt == "mxfp4" else 16
    if fmt == "nvfp4":
        # every block holds its own max, so the dequantized block max is 6 * S_b
        x.reshape(64, -1, bs)[:, :, 0] = np.max(np.abs(x.reshape(64, -1, bs)), axis=2) * 1.0
    # NV: a power-of-two tensor scale keeps G * sb * s_t within bf16's 8 significant bits
    ts = np.float32(2.0 ** -4) if fmt == "nvfp4" else None
    r1 = q(x, fmt=fmt, tensor_scale=ts)
    y = _deq(r1, fmt)
    assert np.all(bf16_to_f32(bf16_bits(y)) == y)          # dequantized values are bf16-exact here
    r2 = q(y, fmt=fmt, tensor_scale=r1["tensor_scale"])
    if fmt == "mxfp4":
        np.testing.assert_array_equal(r2["codes"], r1["codes"])
        np.testing.assert_array_equal(r2["scales"], r1["scales"])
    else:
        c1 = codes_of(r1).reshape(64, -1, bs)
        full = np.any((c1 & 7) == 7, axis=2)               # blocks whose max code is 6
        np.testing.assert_array_equal(codes_of(r2).reshape(64, -1, bs)[full], c1[full])
        np.testing.assert_array_equal(r2["scales"][full], r1["scales"][full])


def _step_local(a):
    return np.where(a <= 2, 0.5, np.where(a <= 4, 1.0, 2.0))


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_half_step_error_bound(fmt):
    rng = np.random.default_rng(5)
    x = (rng.standard_t(3, size=(1000, 1024)) * 0.1).astype(np.float32)
    x = bf16_to_f32(bf16_bits(x))
    r = q(x, fmt=fmt)
    y = _deq(r, fmt).astype(np.float64)
    bs = 32 if fmt == "mxfp4" else 16
    sc = r["scales"]
    if fmt == "mxfp4":
        S = np.ldexp(1.0, sc.astype(np.int64) - 127)
    else:
        S = O.e4m3_decode(sc) * float(r["tensor_scale"])
    S = np.repeat(S, bs, axis=1)
    v = np.abs(x.astype(np.float64)) / S
    err = np.abs(x - y)
    inr = v <= 6
    bound = 0.5 * _step_local(v) * S
    if fmt == "nvfp4":
        bound = bound + np.spacing(np.float32(6.0 * S.max()))      # fp32 division slack
    assert np.all(err[inr] <= bound[inr])
    # saturated MX elements (|v| in (6, 8)) stay within 2 * S
    assert np.all(err[~inr] < 2 * S[~inr])


def test_sr_tensor_level_unbiased_and_deterministic():
    n = 100000
    x = np.full((1, n), 1.3, np.float32)
    x[0, ::32] = 6.0                                       # pin every MX block scale to 2^0
    r1 = q(x, fmt="mxfp4", rnd="sr", seed=9)
    r2 = q(x, fmt="mxfp4", rnd="sr", seed=9)
    r3 = q(x, fmt="mxfp4", rnd="sr", seed=10)
    np.testing.assert_array_equal(r1["codes"], r2["codes"])
    assert not np.array_equal(r1["codes"], r3["codes"])
    y = _deq(r1, "mxfp4")[0]
    mask = np.ones(n, bool)
    mask[::32] = False
    xv = float(bf16_to_f32(bf16_bits(np.array([1.3], np.float32)))[0])
    assert set(np.unique(y[mask])) <= {1.0, 1.5}
    assert abs(y[mask].mean() - xv) <= 5 * 0.5 * np.sqrt(0.36 * 0.64 / mask.sum())


def test_sr_uses_input_index_for_axis0():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((64, 48)).astype(np.float32)
    r0 = q(x, fmt="nvfp4", rnd="sr", seed=77, axis=0)
    # Recompute: element (i, j) of the transposed problem is x[j, i] with index j*48 + i
    xt = bf16_to_f32(bf16_bits(x)).T
    s_t = O.nv_tensor_scale(xt)
    idx = (np.arange(64)[None, :] * 48 + np.arange(48)[:, None]).astype(np.uint64)
    w = O.philox_words(77, idx)
    xb = xt.reshape(48, 4, 16)
    t = ((np.max(np.abs(xb), axis=2) / np.float32(6)).astype(np.float32) / s_t).astype(np.float32)
    sb = O.e4m3_rne_sat(t)
    S = (O.e4m3_decode(sb).astype(np.float32) * s_t).astype(np.float32)
    v = (xb / S[..., None]).astype(np.float32).reshape(48, 64)
    want = O.e2m1_sr(v, w)
    np.testing.assert_array_equal(codes_of(r0), want)


@pytest.mark.parametrize("axis", [0, 1])
@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_sr_row_shards_with_index_base_reproduce_the_whole(fmt, axis):
    """A row shard quantized with idx_base = first_row * cols (and the whole tensor's s_t) draws the
    whole tensor's Philox words, so the shards' codes and scales are the whole's, piece by piece."""
    rng = np.random.default_rng(3)
    x = bf16_to_f32(bf16_bits((rng.standard_t(3, size=(96, 64)) * 0.1).astype(np.float32)))
    whole = O.quantize_values(x, fmt=fmt, axis=axis, rnd="sr", seed=5)
    ts = whole["tensor_scale"]
    cuts = [0, 32, 64, 96]
    for a, b in zip(cuts, cuts[1:]):
        part = O.quantize_values(x[a:b], fmt=fmt, axis=axis, rnd="sr", seed=5, tensor_scale=ts, idx_base=a * 64)
        local = O.quantize_values(x[a:b], fmt=fmt, axis=axis, rnd="sr", seed=5, tensor_scale=ts)
        if axis == 1:
            np.testing.assert_array_equal(part["codes"], whole["codes"][a:b])
            np.testing.assert_array_equal(part["scales"], whole["scales"][a:b])
        else:
            bs = 32 if fmt == "mxfp4" else 16
            np.testing.assert_array_equal(part["codes"], whole["codes"][:, a // 2:b // 2])
            np.testing.assert_array_equal(part["scales"], whole["scales"][:, a // bs:b // bs])
        if a:
            assert not np.array_equal(part["codes"], local["codes"])    # the index base matters


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_axis0_is_axis1_of_transpose_rtn(fmt):
    rng = np.random.default_rng(2)
    x = rng.standard_normal((96, 64)).astype(np.float32)
    a = q(x, fmt=fmt, axis=0)
    b = q(np.ascontiguousarray(x.T), fmt=fmt, axis=1)
    np.testing.assert_array_equal(a["codes"], b["codes"])
    np.testing.assert_array_equal(a["scales"], b["scales"])


def test_dequantize_bf16_is_rne_of_f32():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((16, 64)).astype(np.float32) * 1e-3
    r = q(x, fmt="nvfp4")
    f = O.dequantize(r["codes"], r["scales"], fmt="nvfp4", tensor_scale=r["tensor_scale"])
    b = O.dequantize(r["codes"], r["scales"], fmt="nvfp4", tensor_scale=r["tensor_scale"], out="bf16")
    np.testing.assert_array_equal(b, f.astype(ml_dtypes.bfloat16).view(np.uint16))


@pytest.mark.filterwarnings("ignore:overflow")
def test_mx_dequantize_exact_powers_of_two():
    codes = O.pack_nibbles(np.arange(32, dtype=np.uint8).reshape(1, 32) % 16)
    for byte in (0, 1, 100, 127, 200, 254):
        y = O.dequantize(codes, np.array([[byte]], np.uint8), fmt="mxfp4")
        want = O.e2m1_decode(np.arange(32) % 16) * 2.0 ** (byte - 127)
        np.testing.assert_array_equal(y[0], want.astype(np.float32))
