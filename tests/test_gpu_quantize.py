"""GPU parity: quantize / Hadamard-quantize / dequantize / amax through the C ABI
against the CPU oracle.  Codes, scales and tensor scales must be bit-exact;
rotated values within 1e-6 of the block RMS."""
import numpy as np
import pytest
import torch

import oracle as O
import microscaling_fp4_quantization_mxfp4_b200 as F
from gpu_utils import dev_bf16, host_f32, host_u8, host_bf16_bits, mixed_input
from workloads import bf16_to_f32, nvfp4_student_t

pytestmark = pytest.mark.gpu

SHAPES_AX1 = [(1, 32), (7, 64), (200, 384), (129, 4096), (33, 1056)]
SHAPES_AX0 = [(32, 8), (96, 200), (384, 136), (160, 72)]


def _check_against_oracle(q, ref, fmt, axis, rows, cols, sf):
    np.testing.assert_array_equal(host_u8(q.codes), ref["codes"])
    if sf == "rowmajor":
        np.testing.assert_array_equal(host_u8(q.scales), ref["scales"])
    else:
        np.testing.assert_array_equal(host_u8(q.scales), O.sf_to_mma(ref["scales"]))
    if fmt == "nvfp4":
        assert host_f32(q.tensor_scale)[0] == ref["tensor_scale"]


@pytest.mark.parametrize("sf", ["rowmajor", "mma"])
@pytest.mark.parametrize("rnd", ["rtn", "sr"])
@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("shape", SHAPES_AX1)
def test_quantize_axis1(shape, fmt, rnd, sf):
    rows, cols = shape
    xb = mixed_input(rows, cols, rows * 7 + cols, fmt)
    q = F.fp4_quantize(dev_bf16(xb), fmt=fmt, axis=1, rnd=rnd, seed=1234567890123, sf_layout=sf)
    ref = O.quantize(xb, fmt=fmt, axis=1, rnd=rnd, seed=1234567890123)
    _check_against_oracle(q, ref, fmt, 1, rows, cols, sf)


@pytest.mark.parametrize("sf", ["rowmajor", "mma"])
@pytest.mark.parametrize("rnd", ["rtn", "sr"])
@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("shape", SHAPES_AX0 + [(48, 24)])
def test_quantize_axis0(shape, fmt, rnd, sf):
    rows, cols = shape
    if rows % (32 if fmt == "mxfp4" else 16):
        pytest.skip("rows not a multiple of the block")
    xb = mixed_input(rows, cols, rows * 5 + cols, fmt)
    q = F.fp4_quantize(dev_bf16(xb), fmt=fmt, axis=0, rnd=rnd, seed=42, sf_layout=sf)
    ref = O.quantize(xb, fmt=fmt, axis=0, rnd=rnd, seed=42)
    _check_against_oracle(q, ref, fmt, 0, rows, cols, sf)


@pytest.mark.parametrize("axis", [0, 1])
@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_quantize_strided_input(fmt, axis):
    xb_full = mixed_input(128, 320, 3, fmt)
    xt = dev_bf16(xb_full)[:, :256]                      # ld = 320 > cols = 256
    xb = np.ascontiguousarray(xb_full[:, :256])
    q = F.fp4_quantize(xt, fmt=fmt, axis=axis, rnd="sr", seed=5)
    ref = O.quantize(xb, fmt=fmt, axis=axis, rnd="sr", seed=5)
    _check_against_oracle(q, ref, fmt, axis, 128, 256, "rowmajor")


def test_nv_tensor_scale_in_and_copy_out():
    xb = mixed_input(64, 128, 9, "nvfp4")
    ts = torch.tensor([0.0123], dtype=torch.float32, device="cuda")
    out = torch.zeros(1, dtype=torch.float32, device="cuda")
    q = F.fp4_quantize(dev_bf16(xb), fmt="nvfp4", tensor_scale_in=ts, tensor_scale_out=out)
    ref = O.quantize(xb, fmt="nvfp4", tensor_scale=np.float32(0.0123))
    np.testing.assert_array_equal(host_u8(q.codes), ref["codes"])
    np.testing.assert_array_equal(host_u8(q.scales), ref["scales"])
    assert host_f32(out)[0] == np.float32(0.0123)


def test_sr_deterministic_and_seeded():
    xb = mixed_input(64, 512, 11, "mxfp4")
    x = dev_bf16(xb)
    a = F.fp4_quantize(x, fmt="mxfp4", rnd="sr", seed=7)
    b = F.fp4_quantize(x, fmt="mxfp4", rnd="sr", seed=7)
    c = F.fp4_quantize(x, fmt="mxfp4", rnd="sr", seed=8)
    assert torch.equal(a.codes, b.codes)
    assert not torch.equal(a.codes, c.codes)


SHARD_CASES = [(1, (300, 384), [0, 1, 150, 299, 300]), (1, (2048, 4096), [0, 16, 1000, 2048]),
               (0, (512, 200), [0, 64, 320, 512]), (0, (4096, 1024), [0, 2048, 4096])]


@pytest.mark.parametrize("rnd", ["rtn", "sr"])
@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("axis, shape, cuts", SHARD_CASES)
def test_row_shards_reproduce_the_whole(axis, shape, cuts, fmt, rnd):
    """fp4_quantize_shard on each row shard (NVFP4 under the whole tensor's scale) gives the whole
    tensor's codes and scales bit for bit; each shard also matches the oracle with its index base."""
    rows, cols = shape
    xb = mixed_input(rows, cols, rows + 3 * cols, fmt)
    x = dev_bf16(xb)
    whole = F.fp4_quantize(x, fmt=fmt, axis=axis, rnd=rnd, seed=0x5EED)
    ts = whole.tensor_scale
    for a, b in zip(cuts, cuts[1:]):
        part = F.fp4_quantize(x[a:b], fmt=fmt, axis=axis, rnd=rnd, seed=0x5EED, tensor_scale_in=ts, first_row=a)
        bs = 32 if fmt == "mxfp4" else 16
        if axis == 1:
            assert torch.equal(part.codes, whole.codes[a:b]) and torch.equal(part.scales, whole.scales[a:b])
        else:
            assert torch.equal(part.codes, whole.codes[:, a // 2:b // 2])
            assert torch.equal(part.scales, whole.scales[:, a // bs:b // bs])
    a, b = cuts[1], cuts[2]
    s_t = None if ts is None else host_f32(ts)[0]
    ref = O.quantize(np.ascontiguousarray(xb[a:b]), fmt=fmt, axis=axis, rnd=rnd, seed=0x5EED, tensor_scale=s_t,
                     idx_base=a * cols)
    part = F.fp4_quantize(x[a:b], fmt=fmt, axis=axis, rnd=rnd, seed=0x5EED, tensor_scale_in=ts, first_row=a)
    _check_against_oracle(part, ref, fmt, axis, b - a, cols, "rowmajor")


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_row_shard_far_into_a_tensor(fmt):
    """A shard 2^24 rows into a 4096-column tensor: Philox counters above 2^32 (the high word)."""
    xb = mixed_input(64, 4096, 17, fmt)
    first = 1 << 24
    q = F.fp4_quantize(dev_bf16(xb), fmt=fmt, rnd="sr", seed=99, first_row=first)
    ref = O.quantize(xb, fmt=fmt, rnd="sr", seed=99, idx_base=first * 4096)
    _check_against_oracle(q, ref, fmt, 1, 64, 4096, "rowmajor")


def test_zero_tensor_nv():
    x = torch.zeros((16, 64), dtype=torch.bfloat16, device="cuda")
    q = F.fp4_quantize(x, fmt="nvfp4")
    assert host_f32(q.tensor_scale)[0] == 1.0
    assert int(q.codes.sum()) == 0 and int(q.scales.sum()) == 0


@pytest.mark.parametrize("out", ["f32", "bf16"])
@pytest.mark.parametrize("sf", ["rowmajor", "mma"])
@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_dequantize(fmt, sf, out):
    xb = mixed_input(200, 384, 21, fmt)
    q = F.fp4_quantize(dev_bf16(xb), fmt=fmt, sf_layout=sf)
    y = F.fp4_dequantize(q.codes, q.scales, q.tensor_scale, fmt=fmt, sf_layout=sf, out_dtype=out)
    ref = O.quantize(xb, fmt=fmt)
    want = O.dequantize(ref["codes"], ref["scales"], fmt=fmt, tensor_scale=ref["tensor_scale"], out=out)
    if out == "f32":
        got = host_f32(y)
        np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))
    else:
        np.testing.assert_array_equal(host_bf16_bits(y), want)


def test_dequantize_mx_extreme_scales():
    # every scale byte the quantizer can emit for finite bf16 input, including 2^-127
    codes = torch.arange(256, dtype=torch.int64).remainder(256).to(torch.uint8).reshape(8, 32).cuda()
    sc = torch.tensor([[0, 1], [2, 60], [100, 127], [128, 150], [200, 240], [250, 251], [252, 0], [3, 4]],
                      dtype=torch.uint8, device="cuda")
    y = F.fp4_dequantize(codes, sc, fmt="mxfp4")
    want = O.dequantize(host_u8(codes), host_u8(sc), fmt="mxfp4")
    np.testing.assert_array_equal(host_f32(y).view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("had", [16, 32, 64, 128])
@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_hadamard_quantize(fmt, had):
    rows, cols = 96, 1024
    g = np.random.default_rng(had)
    x = g.standard_normal((rows, cols)).astype(np.float32)
    x[:, g.choice(cols, 10, replace=False)] *= 50.0         # outlier channels
    from workloads import bf16_bits
    xb = bf16_bits(x)
    rot = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    q = F.fp4_hadamard_quantize(dev_bf16(xb), had, fmt=fmt, rotated_out=rot)
    ref = O.quantize(xb, fmt=fmt, had_block=had)
    got_rot = host_f32(rot)
    # rotated values within 1e-6 of the block RMS
    rms = np.sqrt(np.mean(ref["rotated"].astype(np.float64).reshape(rows, -1, had) ** 2, axis=2))
    err = np.abs(got_rot.astype(np.float64) - ref["rotated"]).reshape(rows, -1, had)
    assert np.all(err <= 1e-6 * rms[..., None] + 1e-30)
    # the quantizer applied to the GPU's own rotated values is bit-exact
    ts = None if fmt == "mxfp4" else O.nv_tensor_scale(got_rot)
    ref_gpu_rot = O.quantize_values(got_rot, fmt=fmt, tensor_scale=ts)
    np.testing.assert_array_equal(host_u8(q.codes), ref_gpu_rot["codes"])
    np.testing.assert_array_equal(host_u8(q.scales), ref_gpu_rot["scales"])
    if fmt == "nvfp4":
        assert host_f32(q.tensor_scale)[0] == ts
    # against the oracle's own rotation: at most 1e-4 of codes differ, each by one grid step
    # (positions on the signed grid -6 .. -0.5, 0, 0.5 .. 6, where +0 and -0 are one point)
    gc = O.unpack_nibbles(host_u8(q.codes)).astype(np.int64)
    rc = O.unpack_nibbles(ref["codes"]).astype(np.int64)
    gpos = np.where(gc & 8, -(gc & 7), gc & 7)
    rpos = np.where(rc & 8, -(rc & 7), rc & 7)
    diff = gpos != rpos
    assert diff.mean() <= 1e-4
    assert np.all(np.abs(gpos - rpos) <= 1)


def test_amax_and_tensor_scale():
    xb = mixed_input(300, 264, 17, "nvfp4")
    x = dev_bf16(xb)
    a = F.fp4_amax(x)
    want = np.float32(np.max(np.abs(bf16_to_f32(xb))))
    assert host_f32(a)[0] == want
    ts = F.fp4_nv_tensor_scale(a)
    assert host_f32(ts)[0] == O.nv_tensor_scale(bf16_to_f32(xb))
    z = F.fp4_nv_tensor_scale(torch.zeros(1, device="cuda"))
    assert host_f32(z)[0] == 1.0


@pytest.mark.parametrize("rnd", ["rtn", "sr"])
def test_full_size_nvfp4_student_t_4096(rnd):
    """4096 x 4096 0.1*Student-t(3), seed 1: the full quantize+dequantize case, all outputs
    for RTN; 256 sampled rows (with their global Philox indices) for SR."""
    xb = nvfp4_student_t(4096, 4096, seed=1)
    x = dev_bf16(xb)
    q = F.fp4_quantize(x, fmt="nvfp4", rnd=rnd, seed=1, sf_layout="rowmajor")
    y = F.fp4_dequantize(q.codes, q.scales, q.tensor_scale, fmt="nvfp4")
    x32 = bf16_to_f32(xb)
    s_t = O.nv_tensor_scale(x32)
    assert host_f32(q.tensor_scale)[0] == s_t
    if rnd == "rtn":
        rows = np.arange(4096)
    else:
        rows = np.sort(np.random.default_rng(0).choice(4096, 256, replace=False))
    codes, scales, deq = host_u8(q.codes), host_u8(q.scales), host_f32(y)
    for r0 in range(0, len(rows), 512):
        blk = rows[r0:r0 + 512]
        if rnd == "rtn":
            ref = O.quantize_values(x32[blk], fmt="nvfp4", rnd=rnd, seed=1, tensor_scale=s_t)
            np.testing.assert_array_equal(codes[blk], ref["codes"])
            np.testing.assert_array_equal(scales[blk], ref["scales"])
        else:
            for r in blk:
                ref = O.quantize_values(x32[r:r + 1], fmt="nvfp4", rnd=rnd, seed=1, tensor_scale=s_t,
                                        idx_base=int(r) * 4096)
                np.testing.assert_array_equal(codes[r:r + 1], ref["codes"])
                np.testing.assert_array_equal(scales[r:r + 1], ref["scales"])
        want = O.dequantize(codes[blk], scales[blk], fmt="nvfp4", tensor_scale=s_t)
        np.testing.assert_array_equal(deq[blk].view(np.uint32), want.view(np.uint32))


def test_nv_two_pass_path_large_tensor():
    """A 64 MiB tensor is larger than the SMs' shared memory, so NVFP4 without a given tensor scale
    takes the two-pass path (amax kernel, then quantize); 64 sampled rows checked bit-exactly."""
    from workloads import student_t_bf16
    xb = student_t_bf16((8192, 4096), 3.0, 0.1, 7, 0)
    x = dev_bf16(xb)
    q = F.fp4_quantize(x, fmt="nvfp4", rnd="sr", seed=3)
    x32 = bf16_to_f32(xb)
    s_t = O.nv_tensor_scale(x32)
    assert host_f32(q.tensor_scale)[0] == s_t
    codes, scales = host_u8(q.codes), host_u8(q.scales)
    for r in np.sort(np.random.default_rng(1).choice(8192, 64, replace=False)):
        ref = O.quantize_values(x32[r:r + 1], fmt="nvfp4", rnd="sr", seed=3, tensor_scale=s_t, idx_base=int(r) * 4096)
        np.testing.assert_array_equal(codes[r:r + 1], ref["codes"])
        np.testing.assert_array_equal(scales[r:r + 1], ref["scales"])


def _sr_edge_blocks(rows: int, cols: int, seed: int) -> np.ndarray:
    """MX blocks whose amax (7.5 or 6) fixes the scale at 1, so the scaled values are the inputs:
    zeros of both signs, bf16 subnormals, tiny normals on both sides of 2^-9 (where the fixed-point
    split of the stochastic rounding changes path), every grid point, midpoints, values just
    below 2, 4 and 6, values above 6 (saturating), and random values over many binades."""
    from workloads import bf16_bits
    g = np.random.default_rng(seed)
    edge = np.array([0.0, -0.0, 2.0 ** -133, -2.0 ** -130, 2.0 ** -126, 2.0 ** -11, 2.0 ** -10, 2.0 ** -9,
                     3 * 2.0 ** -10, 2.0 ** -8, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, 0.25, 0.75, 1.25, 1.75,
                     2.5, 3.5, 5.0, 1.9921875, 3.984375, 5.96875, 6.5, 7.0, -7.5, -5.0, -0.001],
                    dtype=np.float32)
    x = np.empty((rows, cols), dtype=np.float32)
    for r in range(rows):
        for b in range(cols // 32):
            if (r + b) % 2 == 0:
                blk = g.permutation(edge).copy()
            else:
                blk = (g.standard_normal(32) * np.exp2(g.integers(-14, 3, 32))).astype(np.float32)
            blk[0] = 7.5 if (r + b) % 3 else 6.0
            x[r, 32 * b:32 * b + 32] = blk
    return bf16_bits(np.clip(x, -7.5, 7.5))


@pytest.mark.parametrize("axis", [1, 0])
@pytest.mark.parametrize("seed", [1, 0xDEADBEEFCAFEF00D])
def test_sr_edge_values_mx(axis, seed):
    """Stochastic rounding at the edges of its arithmetic, bit-exact against the oracle, along
    both axes (axis 0 transposes the edge blocks, so they are built column-wise there)."""
    xb = _sr_edge_blocks(64, 256, seed & 0xFFFF)
    if axis == 0:
        xb = np.ascontiguousarray(xb.T)
    q = F.fp4_quantize(dev_bf16(xb), fmt="mxfp4", axis=axis, rnd="sr", seed=seed)
    ref = O.quantize(xb, fmt="mxfp4", axis=axis, rnd="sr", seed=seed)
    np.testing.assert_array_equal(host_u8(q.scales), ref["scales"])
    np.testing.assert_array_equal(host_u8(q.codes), ref["codes"])
    F.fp4_check_device_errors()


@pytest.mark.parametrize("rnd", ["rtn", "sr"])
@pytest.mark.parametrize("scale", [1.0, 1e-32])
def test_nv_tiny_elements(rnd, scale):
    """NVFP4 blocks holding elements far below the block maximum (down to bf16 subnormals and
    signed zeros), in a tensor of ordinary magnitude (scales S >= 2^-100: the fast division path
    without a per-element test for RTN) and in an all-tiny tensor (S < 2^-100: IEEE division);
    codes and scales bit-exact against the oracle."""
    from workloads import bf16_bits
    g = np.random.default_rng(7)
    x = (g.standard_normal((64, 256)) * scale).astype(np.float32)
    tiny = np.array([1e-35, -1e-35, 2.0 ** -120, -(2.0 ** -126), 2.0 ** -133, -(2.0 ** -133), 0.0, -0.0, 1e-38,
                     2.0 ** -104, -(2.0 ** -103), 2.0 ** -102], dtype=np.float32)
    for r in range(0, 64, 3):
        cols = g.choice(256, 12, replace=False)
        x[r, cols] = tiny
    xb = bf16_bits(x)
    q = F.fp4_quantize(dev_bf16(xb), fmt="nvfp4", rnd=rnd, seed=99)
    ref = O.quantize(xb, fmt="nvfp4", rnd=rnd, seed=99)
    assert host_f32(q.tensor_scale)[0] == ref["tensor_scale"]
    np.testing.assert_array_equal(host_u8(q.scales), ref["scales"])
    np.testing.assert_array_equal(host_u8(q.codes), ref["codes"])
    F.fp4_check_device_errors()


@pytest.mark.parametrize("sf", ["rowmajor", "mma"])
@pytest.mark.parametrize("rnd", ["rtn", "sr"])
@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("shape", [(64, 64), (96, 160), (256, 4096), (4096, 512)])
def test_quantize_2d(shape, fmt, rnd, sf):
    """Square-tile quantization: W's codes/scales along its rows and W^T's along its rows,
    bit-exact against the oracle (tensor-core layout compared after the oracle's permutation)."""
    rows, cols = shape
    bs = 32 if fmt == "mxfp4" else 16
    if rows % bs or cols % bs:
        pytest.skip("shape not a multiple of the tile")
    xb = mixed_input(rows, cols, rows * 3 + cols, fmt)
    q, qt = F.fp4_quantize_2d(dev_bf16(xb), fmt=fmt, rnd=rnd, seed=77, sf_layout=sf)
    ref = O.quantize_2d(xb, fmt=fmt, rnd=rnd, seed=77)
    if fmt == "nvfp4":
        assert host_f32(q.tensor_scale)[0] == ref["tensor_scale"]
    np.testing.assert_array_equal(host_u8(q.codes), ref["codes"])
    np.testing.assert_array_equal(host_u8(qt.codes), ref["codes_t"])
    if sf == "rowmajor":
        np.testing.assert_array_equal(host_u8(q.scales), ref["scales"])
        np.testing.assert_array_equal(host_u8(qt.scales), ref["scales_t"])
    else:
        np.testing.assert_array_equal(host_u8(q.scales), O.sf_to_mma(ref["scales"]))
        np.testing.assert_array_equal(host_u8(qt.scales), O.sf_to_mma(ref["scales_t"]))
    F.fp4_check_device_errors()


def test_quantize_2d_feeds_forward_and_dgrad_gemms():
    """The same 2-D-quantized W serves the forward GEMM (W along K) and the dgrad GEMM (W^T along
    N) without requantization: both against the oracle's fp64 products of the dequantized operands."""
    from workloads import normal_bf16
    M, K, N = 256, 512, 384
    xb = normal_bf16((M, K), 1.0, 5, 0)
    wb = normal_bf16((N, K), 0.02, 5, 1)
    dyb = normal_bf16((M, N), 1e-3, 5, 2)
    qw, qwt = F.fp4_quantize_2d(dev_bf16(wb), fmt="nvfp4", sf_layout="mma")
    qx = F.fp4_quantize(dev_bf16(xb), fmt="nvfp4", sf_layout="mma")
    qdy = F.fp4_quantize(dev_bf16(dyb), fmt="nvfp4", rnd="sr", seed=3, sf_layout="mma")
    y = F.fp4_gemm(qx.codes, qx.scales, qw.codes, qw.scales, fmt="nvfp4", a_tensor_scale=qx.tensor_scale,
                   b_tensor_scale=qw.tensor_scale, out_dtype="f32")
    dx = F.fp4_gemm(qdy.codes, qdy.scales, qwt.codes, qwt.scales, fmt="nvfp4", a_tensor_scale=qdy.tensor_scale,
                    b_tensor_scale=qwt.tensor_scale, out_dtype="f32")
    ow = O.quantize_2d(wb, fmt="nvfp4")
    ox = O.quantize(xb, fmt="nvfp4")
    ody = O.quantize(dyb, fmt="nvfp4", rnd="sr", seed=3)
    yr, bd = O.gemm_ref(ox, {"codes": ow["codes"], "scales": ow["scales"], "tensor_scale": ow["tensor_scale"]},
                        "nvfp4")
    assert np.all(np.abs(host_f32(y) - yr) <= 1e-5 * bd)
    dr, bd2 = O.gemm_ref(ody, {"codes": ow["codes_t"], "scales": ow["scales_t"], "tensor_scale": ow["tensor_scale"]},
                         "nvfp4")
    assert np.all(np.abs(host_f32(dx) - dr) <= 1e-5 * bd2)
    F.fp4_check_device_errors()


def _four_six_check(q, xb, axis, rnd, seed, sf, ts=None):
    """Bit-exact against the oracle's four-over-six, and not vacuous: some block took max->4."""
    ref = O.quantize(xb, fmt="nvfp4_4o6", axis=axis, rnd=rnd, seed=seed, tensor_scale=ts)
    _check_against_oracle(q, ref, "nvfp4", axis, *xb.shape, sf)
    plain = O.quantize(xb, fmt="nvfp4", axis=axis, rnd=rnd, seed=seed, tensor_scale=ts)
    assert np.any(ref["scales"] != plain["scales"])


@pytest.mark.parametrize("sf", ["rowmajor", "mma"])
@pytest.mark.parametrize("rnd", ["rtn", "sr"])
@pytest.mark.parametrize("axis, shape", [(1, (7, 64)), (1, (200, 384)), (1, (129, 4096)), (1, (33, 1056)),
                                         (0, (96, 200)), (0, (384, 136)), (0, (48, 24))])
def test_quantize_four_over_six(axis, shape, rnd, sf):
    """Four-over-six NVFP4 (per block the lower-error of the max->6 and max->4 scales): codes, scales
    and s_t bit-exact, along both axes, both roundings and both scale layouts.  Axis-1 tensors this
    small take the single-pass (fused amax) kernel."""
    rows, cols = shape
    xb = mixed_input(rows, cols, rows * 11 + cols, "nvfp4")
    q = F.fp4_quantize(dev_bf16(xb), fmt="nvfp4_4o6", axis=axis, rnd=rnd, seed=77, sf_layout=sf)
    _four_six_check(q, xb, axis, rnd, 77, sf)
    F.fp4_check_device_errors()


@pytest.mark.parametrize("rnd", ["rtn", "sr"])
def test_quantize_four_over_six_given_scale_and_strided(rnd):
    """The streaming kernel (caller's s_t) and the strided-rows kernel (ld > cols)."""
    xb_full = mixed_input(256, 640, 5, "nvfp4")
    xb = np.ascontiguousarray(xb_full[:, :512])
    ts = np.float32(O.nv_tensor_scale(bf16_to_f32(xb)) * np.float32(1.5))
    ts_dev = torch.tensor([ts], dtype=torch.float32, device="cuda")
    q = F.fp4_quantize(dev_bf16(xb), fmt="nvfp4_4o6", rnd=rnd, seed=9, tensor_scale_in=ts_dev)
    _four_six_check(q, xb, 1, rnd, 9, "rowmajor", ts=ts)
    q2 = F.fp4_quantize(dev_bf16(xb_full)[:, :512], fmt="nvfp4_4o6", rnd=rnd, seed=9, sf_layout="mma")
    _four_six_check(q2, xb, 1, rnd, 9, "mma")
    F.fp4_check_device_errors()


def test_quantize_four_over_six_two_pass_large_tensor():
    """A 64 MiB tensor takes the amax kernel then the streaming four-over-six kernel; 64 sampled rows
    checked bit-exactly against the oracle with the whole tensor's s_t."""
    from workloads import student_t_bf16
    xb = student_t_bf16((8192, 4096), 3.0, 0.1, 7, 0)
    q = F.fp4_quantize(dev_bf16(xb), fmt="nvfp4_4o6", rnd="sr", seed=3)
    x32 = bf16_to_f32(xb)
    s_t = O.nv_tensor_scale(x32)
    assert host_f32(q.tensor_scale)[0] == s_t
    codes, scales = host_u8(q.codes), host_u8(q.scales)
    for r in np.sort(np.random.default_rng(2).choice(8192, 64, replace=False)):
        ref = O.quantize_values(x32[r:r + 1], fmt="nvfp4_4o6", rnd="sr", seed=3, tensor_scale=s_t,
                                idx_base=int(r) * 4096)
        np.testing.assert_array_equal(codes[r:r + 1], ref["codes"])
        np.testing.assert_array_equal(scales[r:r + 1], ref["scales"])


def test_four_over_six_feeds_nvfp4_gemm():
    """Four-over-six outputs are ordinary NVFP4 operands for the block-scaled GEMM."""
    from workloads import normal_bf16
    M, K, N = 256, 512, 384
    xb = normal_bf16((M, K), 1.0, 6, 0)
    wb = normal_bf16((N, K), 0.02, 6, 1)
    qx = F.fp4_quantize(dev_bf16(xb), fmt="nvfp4_4o6", sf_layout="mma")
    qw = F.fp4_quantize(dev_bf16(wb), fmt="nvfp4_4o6", sf_layout="mma")
    y = F.fp4_gemm(qx.codes, qx.scales, qw.codes, qw.scales, fmt="nvfp4", a_tensor_scale=qx.tensor_scale,
                   b_tensor_scale=qw.tensor_scale, out_dtype="f32")
    ox, ow = O.quantize(xb, fmt="nvfp4_4o6"), O.quantize(wb, fmt="nvfp4_4o6")
    yr, bd = O.gemm_ref(ox, ow, "nvfp4")
    assert np.all(np.abs(host_f32(y) - yr) <= 1e-5 * bd)
    F.fp4_check_device_errors()


def _tie_blocks(nblocks: int, seed: int) -> np.ndarray:
    """fp32 [nblocks, 16] blocks whose two four-over-six candidates have exactly equal errors under
    s_t = 1: all +-24 (both exact: 24/4 = 6 on the 6-grid, 24/6 = 4 on the 4-grid) or 24 with +-5
    elsewhere (5/4 = 1.25 ties to 1 -> error 1; 5/6 -> 1 -> error 1)."""
    g = np.random.default_rng(seed)
    x = np.full((nblocks, 16), 24.0, dtype=np.float32)
    x[1::2, 1:] = 5.0
    return x * np.where(g.random((nblocks, 16)) < 0.5, -1.0, 1.0).astype(np.float32)


@pytest.mark.parametrize("rnd", ["rtn", "sr"])
def test_four_over_six_ties_and_extreme_magnitudes(rnd):
    """Blocks the kernels cannot decide in fp32 and settle with the fp64 sums: exact ties (keep the
    max->6 scale), error sums that underflow fp32 (values near 1e-30) or overflow it (near 1e30),
    plus Student-t blocks, some of which tie naturally.  Bit-exact against the oracle."""
    from workloads import bf16_bits, student_t_bf16
    ties = bf16_bits(_tie_blocks(256, 3).reshape(64, 64))
    xb = np.concatenate([ties, student_t_bf16((448, 64), 3.0, 0.1, 8, 0)], axis=0)
    x32 = bf16_to_f32(xb)
    ts = torch.ones(1, dtype=torch.float32, device="cuda")
    q = F.fp4_quantize(dev_bf16(xb), fmt="nvfp4_4o6", rnd=rnd, seed=5, tensor_scale_in=ts)
    ref = O.quantize(xb, fmt="nvfp4_4o6", rnd=rnd, seed=5, tensor_scale=np.float32(1.0))
    _check_against_oracle(q, ref, "nvfp4", 1, *xb.shape, "rowmajor")
    plain = O.quantize(xb, fmt="nvfp4", rnd=rnd, seed=5, tensor_scale=np.float32(1.0))
    np.testing.assert_array_equal(ref["scales"][:64], plain["scales"][:64])          # ties keep max->6
    from oracle.four_over_six import nv_block_candidates, _rtn_sq_error
    xs = x32[64:].reshape(-1, 16)
    sb6, sb4 = nv_block_candidates(np.max(np.abs(xs), axis=-1), np.float32(1.0))
    live = (sb4 != sb6) & (sb4 != 0)
    assert np.any(live & (_rtn_sq_error(xs, sb6, np.float32(1.0)) == _rtn_sq_error(xs, sb4, np.float32(1.0))))
    for mult in (1e-30, 1e30):                       # squared errors far outside fp32's range
        xe = student_t_bf16((128, 256), 3.0, mult, 9, 1)
        q = F.fp4_quantize(dev_bf16(xe), fmt="nvfp4_4o6", rnd=rnd, seed=6)
        _four_six_check(q, xe, 1, rnd, 6, "rowmajor")
    F.fp4_check_device_errors()


# ------------------------------------------------------------ MSE-fitted grid scales ---

@pytest.mark.parametrize("axis", [1, 0])
@pytest.mark.parametrize("rnd", ["rtn", "sr"])
def test_quantize_mxfp4_clip_threshold(axis, rnd):
    """MXFP4 with the MSE-fitted exponent clip threshold 7.25: codes and scales bit-exact, and the
    threshold changes some block exponents against the OCP rule."""
    rows, cols = 96, 256
    xb = mixed_input(rows, cols, 501 + axis, "mxfp4")
    q = F.fp4_quantize(dev_bf16(xb), fmt="mxfp4_gs", axis=axis, rnd=rnd, seed=5, sf_layout="mma")
    ref = O.quantize(xb, fmt="mxfp4_gs", axis=axis, rnd=rnd, seed=5)
    _check_against_oracle(q, ref, "mxfp4", axis, rows, cols, "mma")
    assert np.any(ref["scales"] != O.quantize(xb, fmt="mxfp4", axis=axis, rnd=rnd, seed=5)["scales"])
    F.fp4_check_device_errors()


def test_hadamard_quantize_mxfp4_clip_threshold():
    """The fixed grid scale is meant for MXFP4 behind block-Hadamard rotations: the quantizer applied
    to the kernel's own rotated values is bit-exact (as for the other Hadamard parity tests)."""
    rows, cols = 64, 1024
    g = np.random.default_rng(77)
    from workloads import bf16_bits
    x = g.standard_normal((rows, cols)).astype(np.float32)
    x[:, g.choice(cols, 10, replace=False)] *= 50.0
    xb = bf16_bits(x)
    rot = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    q = F.fp4_hadamard_quantize(dev_bf16(xb), 128, fmt="mxfp4_gs", rotated_out=rot)
    ref = O.quantize_values(host_f32(rot), fmt="mxfp4_gs")
    np.testing.assert_array_equal(host_u8(q.codes), ref["codes"])
    np.testing.assert_array_equal(host_u8(q.scales), ref["scales"])
    F.fp4_check_device_errors()


@pytest.mark.parametrize("shape, iters, rnd, sf", [
    ((64, 256), 0, "rtn", "rowmajor"), ((64, 256), 0, "sr", "mma"), ((64, 256), 2, "rtn", "mma"),
    ((200, 384), 1, "sr", "rowmajor"), ((200, 384), 1, "rtn", "mma"), ((7, 64), 1, "rtn", "rowmajor"),
    ((129, 1024), 1, "sr", "mma")])
def test_quantize_mse(shape, iters, rnd, sf):
    """NVFP4 with MSE-searched block and tensor scales: codes, scales and s_t bit-exact."""
    rows, cols = shape
    xb = student_t_bf16_(shape, 40 + rows)
    q = F.fp4_quantize_mse(dev_bf16(xb), rnd=rnd, seed=11, iters=iters, sf_layout=sf)
    ref = O.quantize_mse(xb, rnd=rnd, seed=11, iters=iters)
    _check_against_oracle(q, ref, "nvfp4", 1, rows, cols, sf)
    F.fp4_check_device_errors()


def student_t_bf16_(shape, seed):
    from workloads import student_t_bf16
    return student_t_bf16(shape, 3.0, 0.1, seed, 0)


def test_quantize_mse_strided_and_tied_blocks():
    """Strided rows (ld > cols) and blocks whose candidates tie exactly -- constant magnitudes exact
    under several bytes, a block exact on a non-standard grid, zero and tiny blocks -- which the
    kernel settles with exact fp64 errors in tie-break order."""
    from workloads import bf16_bits
    g = np.random.default_rng(9)
    x = (g.standard_t(3, size=(32, 320)) * 0.1).astype(np.float32)
    x[0, :16] = 0.65625                               # 2688 * 2^-12 (exact on the 6-grid)
    x[1, :16] = np.float32(2.0 ** -6) * np.array([0, .5, 1, 1.5, 2, 3, 4, 4, -.5, -1, -2, -3, 1.5, .5, 3, -4])
    x[2, :32] = np.where(g.random(32) < 0.5, -1.0, 1.0) * np.float32(0.125)   # +-c: exact under several bytes
    x[3, :16] = 0.0
    x[4, :16] = np.float32(1e-30)
    xb = bf16_bits(x)
    xt = dev_bf16(xb)[:, :256]
    q = F.fp4_quantize_mse(xt, rnd="rtn", iters=1, sf_layout="mma")
    ref = O.quantize_mse(np.ascontiguousarray(xb[:, :256]), rnd="rtn", iters=1)
    _check_against_oracle(q, ref, "nvfp4", 1, 32, 256, "mma")
    F.fp4_check_device_errors()


def test_quantize_mse_full_size_properties():
    """W[1024, 1024] ~ N(0, 0.02) with one tensor step (multi-CTA objective, grid-stride blocks):
    the searched s_t is one of the 17 candidates of amax/2688, its exact objective is no larger than
    that of amax/2688 itself, and 64 sampled rows carry the oracle's bytes and codes under it."""
    from oracle import mse_grid as M
    from workloads import normal_bf16
    xb = normal_bf16((1024, 1024), 0.02, 42, 0)
    q = F.fp4_quantize_mse(dev_bf16(xb), iters=1)
    x32 = bf16_to_f32(xb)
    s0 = O.nv_tensor_scale(x32)
    s1 = host_f32(q.tensor_scale)[0]
    assert s1 in set(M.tensor_candidates(s0).tolist())
    x16 = x32.reshape(-1, 16)
    P = M.objective_exponent(np.float32(np.max(np.abs(x32))))
    assert M.tensor_objective(x16, M.block_step(x16, s1), s1, P) <= M.tensor_objective(x16, M.block_step(x16, s0), s0, P)
    codes, scales = host_u8(q.codes), host_u8(q.scales)
    for r in np.sort(np.random.default_rng(3).choice(1024, 64, replace=False)):
        sb = M.block_step(x32[r].reshape(-1, 16), np.float32(s1))
        np.testing.assert_array_equal(scales[r], sb)
        S = (O.e4m3_decode(sb).astype(np.float32) * np.float32(s1)).astype(np.float32)
        v = (x32[r].reshape(-1, 16) / S[:, None]).astype(np.float32)
        c = np.where((sb == 0)[:, None], np.uint8(0), O.e2m1_rtn(v))
        np.testing.assert_array_equal(codes[r], O.pack_nibbles(c.reshape(1, -1))[0])
    F.fp4_check_device_errors()


# ------------------------------------------------------------- quantize + dequantize ---

@pytest.mark.parametrize("out", ["f32", "bf16"])
@pytest.mark.parametrize("sf", ["rowmajor", "mma"])
@pytest.mark.parametrize("rnd", ["rtn", "sr"])
@pytest.mark.parametrize("fmt, shape, given_ts, strided", [
    ("nvfp4", (200, 384), False, False),        # single-pass amax + quantize kernel
    ("nvfp4", (3, 320), False, False),          # single-pass kernel, a partial tile
    ("nvfp4", (129, 1024), True, False),        # streaming kernel under a caller's s_t
    ("nvfp4", (64, 256), False, True),          # strided rows (ld > cols): amax pass + rows kernel
    ("mxfp4", (96, 512), False, False),
    ("mxfp4_gs", (33, 1056), False, True)])
def test_quantize_dequantize(fmt, shape, given_ts, strided, rnd, sf, out):
    """One launch writes codes, scales and the dequantized values: codes and scales bit-exact
    against the oracle's quantize, values bit-exact against the oracle's dequantize of them."""
    rows, cols = shape
    xfull = mixed_input(rows, cols + (64 if strided else 0), rows + cols, "mxfp4" if fmt != "nvfp4" else "nvfp4")
    xb = np.ascontiguousarray(xfull[:, :cols])
    x = dev_bf16(xfull)[:, :cols] if strided else dev_bf16(xb)
    ts = None
    kw = {}
    if given_ts:
        ts = np.float32(O.nv_tensor_scale(bf16_to_f32(xb)) * np.float32(0.75))
        kw["tensor_scale_in"] = torch.tensor([ts], dtype=torch.float32, device="cuda")
    q, y = F.fp4_quantize_dequantize(x, fmt=fmt, rnd=rnd, seed=21, sf_layout=sf, out_dtype=out, **kw)
    ref = O.quantize(xb, fmt=fmt, rnd=rnd, seed=21, tensor_scale=ts)
    _check_against_oracle(q, ref, "nvfp4" if fmt == "nvfp4" else "mxfp4", 1, rows, cols, sf)
    base = "nvfp4" if fmt == "nvfp4" else "mxfp4"
    want = O.dequantize(ref["codes"], ref["scales"], fmt=base, tensor_scale=ref["tensor_scale"], out=out)
    if out == "f32":
        np.testing.assert_array_equal(host_f32(y).view(np.uint32), want.view(np.uint32))
    else:
        np.testing.assert_array_equal(host_bf16_bits(y), want)
    F.fp4_check_device_errors()


def test_quantize_dequantize_two_pass_large_tensor():
    """A 64 MiB tensor (amax pass, then the streaming kernel): 64 sampled rows bit-exact."""
    from workloads import student_t_bf16
    xb = student_t_bf16((8192, 4096), 3.0, 0.1, 7, 1)
    q, y = F.fp4_quantize_dequantize(dev_bf16(xb), fmt="nvfp4", rnd="sr", seed=4)
    x32 = bf16_to_f32(xb)
    s_t = O.nv_tensor_scale(x32)
    assert host_f32(q.tensor_scale)[0] == s_t
    codes, scales, yv = host_u8(q.codes), host_u8(q.scales), host_f32(y)
    for r in np.sort(np.random.default_rng(5).choice(8192, 64, replace=False)):
        ref = O.quantize_values(x32[r:r + 1], fmt="nvfp4", rnd="sr", seed=4, tensor_scale=s_t, idx_base=int(r) * 4096)
        np.testing.assert_array_equal(codes[r:r + 1], ref["codes"])
        np.testing.assert_array_equal(scales[r:r + 1], ref["scales"])
        want = O.dequantize(ref["codes"], ref["scales"], fmt="nvfp4", tensor_scale=s_t)
        np.testing.assert_array_equal(yv[r:r + 1].view(np.uint32), want.view(np.uint32))
    F.fp4_check_device_errors()


@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_quantize_dequantize_output_16_byte_aligned(out):
    """An output 16- but not 32-byte aligned takes the 16-byte stores: same values."""
    rows, cols = 64, 512
    xb = mixed_input(rows, cols, 77, "nvfp4")
    dt = torch.float32 if out == "f32" else torch.bfloat16
    shift = 4 if out == "f32" else 8                      # 16 bytes
    buf = torch.empty(rows * cols + shift, dtype=dt, device="cuda")
    y = buf[shift:].view(rows, cols)
    q, _ = F.fp4_quantize_dequantize(dev_bf16(xb), fmt="nvfp4", rnd="sr", seed=3, out_dtype=out, out=y)
    ref = O.quantize(xb, fmt="nvfp4", rnd="sr", seed=3)
    want = O.dequantize(ref["codes"], ref["scales"], fmt="nvfp4", tensor_scale=ref["tensor_scale"], out=out)
    got = host_f32(y).view(np.uint32) if out == "f32" else host_bf16_bits(y)
    np.testing.assert_array_equal(got, want.view(np.uint32) if out == "f32" else want)
    F.fp4_check_device_errors()
