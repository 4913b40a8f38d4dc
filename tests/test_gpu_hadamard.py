"""GPU parity of the block-Hadamard-fused quantizer (fp4_hadamard_quantize) against the oracle.

"Bridging the Gap Between Promise and Performance for Microscaling FP4 Quantization", Abstract:
block-wise Hadamard rotations computed online for the activations; its summary post, item 3:
block-diagonal rotations.  The acceptance reading for rotated quantization:
  * rotated values within 1e-6 of the block RMS of the oracle's fp64 rotation;
  * the oracle applied to the kernel's own rotated values gives the kernel's codes and scales bit
    for bit (Philox words at each element's row-major index in the input);
  * against the oracle's own rotation, at most 1e-4 of the codes differ, each by one grid step,
    outside the blocks whose scale sits within 1e-6 (relative) of a scale-rounding boundary, where
    the two fp32 roundings of the rotation may legitimately pick different scales.
Covered here: stochastic rounding for every block size, both formats and both scale layouts;
NVFP4 with a caller's tensor scale; strided rows (ld > cols); and the full 8192 x 4096 activation
tensor with 1% of its channels x50 on sampled rows, which spans several rounds of the streaming
kernel's shared-memory ring.
"""
import numpy as np
import pytest
import torch

import oracle as O
import microscaling_fp4_quantization_mxfp4_b200 as F
from gpu_utils import dev_bf16, host_f32, host_u8
from workloads import bf16_bits, bf16_to_f32, hadamard_acts

pytestmark = pytest.mark.gpu

HADS = [16, 32, 64, 128]
BLOCK = {"mxfp4": 32, "nvfp4": 16}


def _scales_rowmajor(q, sf, out_rows, groups):
    s = host_u8(q.scales)
    return s.reshape(out_rows, groups) if sf == "rowmajor" else O.sf_from_mma(s, out_rows, groups)


def _near_scale_boundary(rot32, fmt, s_t):
    """[n, L/block] mask of blocks whose scale would change under a 1e-6 relative change of the
    block maximum (MX: a power-of-two boundary; NV: an E4M3 rounding midpoint of t)."""
    bs = BLOCK[fmt]
    n, L = rot32.shape
    am = np.max(np.abs(rot32.reshape(n, L // bs, bs).astype(np.float64)), axis=2)
    lo, hi = am * (1 - 1e-6), am * (1 + 1e-6)
    if fmt == "mxfp4":
        return O.mx_scale_exponent(lo.astype(np.float32)) != O.mx_scale_exponent(hi.astype(np.float32))
    t_lo = (lo / 6.0 / np.float64(s_t)).astype(np.float32)
    t_hi = (hi / 6.0 / np.float64(s_t)).astype(np.float32)
    return O.e4m3_rne_sat(t_lo) != O.e4m3_rne_sat(t_hi)


def _quantize_rows(vals32, rows, cols, fmt, rnd, seed, s_t):
    """The oracle on fp32 values of the input rows `rows` (global indices, for the Philox words)."""
    if rnd == "rtn":
        return O.quantize_values(vals32, fmt=fmt, rnd=rnd, seed=seed, tensor_scale=s_t)
    codes, scales = [], []
    for i, r in enumerate(rows):
        ref = O.quantize_values(vals32[i:i + 1], fmt=fmt, rnd=rnd, seed=seed, tensor_scale=s_t,
                                idx_base=int(r) * cols)
        codes.append(ref["codes"])
        scales.append(ref["scales"])
    return {"codes": np.concatenate(codes), "scales": np.concatenate(scales)}


def check_rotated_quantization(codes, scales, got_rot, x_bits, rows, cols, fmt, had, rnd, seed,
                               s_t_kernel, s_t_oracle):
    """codes, scales (row-major), got_rot (fp32 rotated values) and x_bits (bf16 input) of the
    input rows `rows`; s_t_* the NVFP4 tensor scale each side quantizes under (None for MX)."""
    ref_rot = O.block_hadamard(bf16_to_f32(x_bits), had)                     # fp64
    rms = np.sqrt(np.mean(ref_rot.reshape(len(rows), -1, had) ** 2, axis=2))
    err = np.abs(got_rot.astype(np.float64) - ref_rot).reshape(len(rows), -1, had)
    assert np.all(err <= 1e-6 * rms[..., None] + 1e-30), float(np.max(err / (rms[..., None] + 1e-30)))
    # the oracle on the kernel's own rotated values: bit-exact
    mine = _quantize_rows(got_rot, rows, cols, fmt, rnd, seed, s_t_kernel)
    np.testing.assert_array_equal(codes, mine["codes"])
    np.testing.assert_array_equal(scales, mine["scales"])
    # against the oracle's own rotation: at most 1e-4 of codes off, each by one grid step
    ref32 = ref_rot.astype(np.float32)
    theirs = _quantize_rows(ref32, rows, cols, fmt, rnd, seed, s_t_oracle)
    near = _near_scale_boundary(ref32, fmt, s_t_oracle if fmt == "nvfp4" else None)
    keep = ~near
    np.testing.assert_array_equal(scales[keep], theirs["scales"][keep])
    bs = BLOCK[fmt]
    gc = O.unpack_nibbles(codes).astype(np.int64).reshape(len(rows), -1, bs)
    rc = O.unpack_nibbles(theirs["codes"]).astype(np.int64).reshape(len(rows), -1, bs)
    gpos = np.where(gc & 8, -(gc & 7), gc & 7)[keep]
    rpos = np.where(rc & 8, -(rc & 7), rc & 7)[keep]
    assert np.mean(gpos != rpos) <= 1e-4
    assert np.all(np.abs(gpos - rpos) <= 1)
    return int(near.sum())


def _acts(rows, cols, seed, outliers=10):
    g = np.random.default_rng(seed)
    x = g.standard_normal((rows, cols)).astype(np.float32)
    x[:, g.choice(cols, outliers, replace=False)] *= 50.0
    return bf16_bits(x)


@pytest.mark.parametrize("sf", ["rowmajor", "mma"])
@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("had", HADS)
def test_hadamard_quantize_sr(had, fmt, sf):
    """Stochastic rounding after the rotation, every block size, both formats and layouts."""
    rows, cols, seed = 320, 4096, 0xC0FFEE + had
    xb = _acts(rows, cols, had * 3 + (fmt == "nvfp4"))
    rot = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    q = F.fp4_hadamard_quantize(dev_bf16(xb), had, fmt=fmt, rnd="sr", seed=seed, sf_layout=sf, rotated_out=rot)
    got_rot = host_f32(rot)
    s_k = s_o = None
    if fmt == "nvfp4":
        s_k = O.nv_tensor_scale(got_rot)
        s_o = O.nv_tensor_scale(O.block_hadamard(bf16_to_f32(xb), had).astype(np.float32))
        assert host_f32(q.tensor_scale)[0] == s_k
    rows_idx = np.arange(rows)
    check_rotated_quantization(host_u8(q.codes), _scales_rowmajor(q, sf, rows, cols // BLOCK[fmt]), got_rot, xb,
                               rows_idx, cols, fmt, had, "sr", seed, s_k, s_o)
    F.fp4_check_device_errors()


@pytest.mark.parametrize("rnd", ["rtn", "sr"])
@pytest.mark.parametrize("had", HADS)
def test_hadamard_quantize_nvfp4_given_tensor_scale(had, rnd):
    """NVFP4 under a caller's tensor scale (contiguous rows: the streaming kernel), which is also
    copied to tensor_scale_out."""
    rows, cols = 200, 2048
    xb = _acts(rows, cols, 50 + had)
    ts = torch.tensor([0.0213], dtype=torch.float32, device="cuda")
    ts_out = torch.zeros(1, dtype=torch.float32, device="cuda")
    rot = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    q = F.fp4_hadamard_quantize(dev_bf16(xb), had, fmt="nvfp4", rnd=rnd, seed=77, tensor_scale_in=ts,
                                tensor_scale_out=ts_out, rotated_out=rot)
    assert host_f32(ts_out)[0] == np.float32(0.0213)
    s = np.float32(0.0213)
    check_rotated_quantization(host_u8(q.codes), host_u8(q.scales), host_f32(rot), xb, np.arange(rows), cols,
                               "nvfp4", had, rnd, 77, s, s)


@pytest.mark.parametrize("rnd", ["rtn", "sr"])
@pytest.mark.parametrize("fmt, given", [("mxfp4", False), ("nvfp4", False), ("nvfp4", True)])
@pytest.mark.parametrize("had", HADS)
def test_hadamard_quantize_strided_rows(had, fmt, given, rnd):
    """Rows with ld > cols (the strided-row kernel), with the rotation dump of the visible columns;
    NVFP4 with its own amax pass or a caller's tensor scale."""
    rows, cols, ld = 136, 1024, 1280
    full = _acts(rows, ld, 90 + had)
    xt = dev_bf16(full)[:, :cols]
    xb = np.ascontiguousarray(full[:, :cols])
    rot = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    ts = torch.tensor([0.0377], dtype=torch.float32, device="cuda") if given else None
    q = F.fp4_hadamard_quantize(xt, had, fmt=fmt, rnd=rnd, seed=5, tensor_scale_in=ts, rotated_out=rot)
    got_rot = host_f32(rot)
    s_k = s_o = None
    if fmt == "nvfp4":
        if given:
            s_k = s_o = np.float32(0.0377)
        else:
            s_k = O.nv_tensor_scale(got_rot)
            s_o = O.nv_tensor_scale(O.block_hadamard(bf16_to_f32(xb), had).astype(np.float32))
        assert host_f32(q.tensor_scale)[0] == s_k
    check_rotated_quantization(host_u8(q.codes), host_u8(q.scales), got_rot, xb, np.arange(rows), cols, fmt, had,
                               rnd, 5, s_k, s_o)


@pytest.fixture(scope="module")
def cfg3_acts():
    """X[8192, 4096] ~ N(0,1) with 41 channels x50 (the Hadamard-rotated activation workload)."""
    xb = hadamard_acts(8192, 4096, seed=2)
    return xb, dev_bf16(xb)


def _oracle_rot_amax(xb, had):
    x = bf16_to_f32(xb)
    m = np.float32(0.0)
    for r0 in range(0, x.shape[0], 1024):
        m = max(m, np.float32(np.max(np.abs(O.block_hadamard(x[r0:r0 + 1024], had).astype(np.float32)))))
    return m


@pytest.mark.parametrize("fmt, rnd", [("mxfp4", "rtn"), ("nvfp4", "rtn"), ("mxfp4", "sr"), ("nvfp4", "sr")])
@pytest.mark.parametrize("had", HADS)
def test_hadamard_quantize_full_size_8192x4096(cfg3_acts, had, fmt, rnd):
    """The full activation tensor, tensor-core scale layout as the GEMM consumes it; 256 rows
    spread over the tensor checked against the oracle (NVFP4: the tensor scale over all rows)."""
    xb, x = cfg3_acts
    rows, cols = x.shape
    rot = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    seed = 2024 + had
    q = F.fp4_hadamard_quantize(x, had, fmt=fmt, rnd=rnd, seed=seed, sf_layout="mma", rotated_out=rot)
    sample = np.sort(np.random.default_rng(had + 7).choice(rows, 256, replace=False))
    sel = torch.from_numpy(sample).cuda()
    got_rot = host_f32(rot[sel])
    s_k = s_o = None
    if fmt == "nvfp4":
        amax_k = np.float32(rot.abs().max().item())
        s_k = np.float32(amax_k / np.float32(2688.0))
        s_o = np.float32(_oracle_rot_amax(xb, had) / np.float32(2688.0))
        assert host_f32(q.tensor_scale)[0] == s_k
    scales = O.sf_from_mma(host_u8(q.scales), rows, cols // BLOCK[fmt])[sample]
    near = check_rotated_quantization(host_u8(q.codes[sel]), scales, got_rot, xb[sample], sample, cols, fmt, had,
                                      rnd, seed, s_k, s_o)
    assert near <= 64
    F.fp4_check_device_errors()


@pytest.mark.parametrize("sf", ["rowmajor", "mma"])
@pytest.mark.parametrize("had", HADS)
def test_hadamard_mxfp4_rtn_without_rotation_dump(had, sf):
    """The production call (no dump of the rotated values) gives the codes and scales of the call
    with the dump, which the other tests pin to the oracle, over rows scaled from 2^-130 to 2^121
    (subnormal quotients, block maxima at and above 2^125), for the streaming and the strided-row
    kernels."""
    rows, cols = 512, 1024
    g = np.random.default_rng(500 + had)
    x = g.standard_normal((rows, cols)).astype(np.float32)
    x *= np.exp2(g.integers(-130, 122, size=(rows, 1))).astype(np.float32)
    x[:8] = (g.standard_normal((8, cols)) * np.float32(2.0 ** 121)).astype(np.float32)   # maxima >= 2^125
    x[8:16, ::5] *= np.float32(2.0 ** -40)                                                # tiny inside blocks
    xb = bf16_bits(x)
    assert np.all(np.isfinite(bf16_to_f32(xb)))
    xd = dev_bf16(xb)
    rot = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    q_dump = F.fp4_hadamard_quantize(xd, had, fmt="mxfp4", sf_layout=sf, rotated_out=rot)
    q_fold = F.fp4_hadamard_quantize(xd, had, fmt="mxfp4", sf_layout=sf)
    np.testing.assert_array_equal(host_u8(q_fold.codes), host_u8(q_dump.codes))
    np.testing.assert_array_equal(host_u8(q_fold.scales), host_u8(q_dump.scales))
    ref = O.quantize_values(host_f32(rot), fmt="mxfp4")
    np.testing.assert_array_equal(host_u8(q_fold.codes), ref["codes"])
    # the strided-row kernel (ld > cols) folds the same way
    wide = torch.zeros((rows, cols + 64), dtype=torch.bfloat16, device="cuda")
    wide[:, :cols] = xd
    q_strided = F.fp4_hadamard_quantize(wide[:, :cols], had, fmt="mxfp4", sf_layout=sf)
    np.testing.assert_array_equal(host_u8(q_strided.codes), host_u8(q_dump.codes))
    np.testing.assert_array_equal(host_u8(q_strided.scales), host_u8(q_dump.scales))
    F.fp4_check_device_errors()
