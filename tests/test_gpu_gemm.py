"""GPU parity: the tcgen05 block-scaled FP4 GEMM through the C ABI against the
oracle's fp64 reference: |dY| <= 1e-5 * sum_k |alpha a b| per element (fp32
output); bf16 output = RNE_bf16 of the fp32 output within one bf16 ulp."""
import numpy as np
import pytest
import torch

import oracle as O
import microscaling_fp4_quantization_mxfp4_b200 as F
from gpu_utils import dev_bf16, host_f32, host_u8, mixed_input
from workloads import (bf16_to_f32, hadamard_acts, hadamard_weights, llama_acts, llama_weights,
                       mx_linear_128x512, vit_layer, normal_bf16)

pytestmark = pytest.mark.gpu

TOL = 1e-5


def _gpu_quant(x_dev, fmt, axis=1, rnd="rtn", seed=0):
    return F.fp4_quantize(x_dev, fmt=fmt, axis=axis, rnd=rnd, seed=seed, sf_layout="mma")


def _as_oracle(q, fmt, rows, k):
    """GPU quantizer output -> oracle operand dict (scales read back from the tensor-core layout)."""
    bs = 32 if fmt == "mxfp4" else 16
    d = {"codes": host_u8(q.codes), "scales": O.sf_from_mma(host_u8(q.scales), rows, k // bs)}
    d["tensor_scale"] = None if q.tensor_scale is None else host_f32(q.tensor_scale)[0]
    return d


def _check(y_gpu, y_ref, bound):
    err = np.abs(y_gpu.astype(np.float64) - y_ref)
    bad = err > TOL * bound
    assert not bad.any(), f"{bad.sum()} elements out of tolerance; worst ratio {np.max(err / np.maximum(bound, 1e-300))}"


def _bf16_ulp_check(y_bf16, y_f32):
    want = y_f32.astype(np.float32)
    got = y_bf16.float().cpu().numpy().astype(np.float64)
    ref = torch.from_numpy(want).to(torch.bfloat16).float().numpy().astype(np.float64)
    ulp = np.abs(np.spacing(ref.astype(np.float32)).astype(np.float64)) * 2 ** 16   # bf16 ulp at ref
    assert np.all(np.abs(got - ref) <= ulp + 1e-45)


def test_mx_linear_128x512():
    """X[128,512] ~ N(0,1), W[512,512] ~ N(0,0.02), MXFP4 RTN along K, Y = deq(X) deq(W)^T in fp32."""
    xb, wb = mx_linear_128x512(0)
    qx, qw = _gpu_quant(dev_bf16(xb), "mxfp4"), _gpu_quant(dev_bf16(wb), "mxfp4")
    y = F.fp4_gemm(qx.codes, qx.scales, qw.codes, qw.scales, fmt="mxfp4", out_dtype="f32")
    ox = O.quantize(xb, fmt="mxfp4")
    ow = O.quantize(wb, fmt="mxfp4")
    # the GPU operands equal the oracle's (quantize parity), so the reference uses the oracle's
    np.testing.assert_array_equal(_as_oracle(qx, "mxfp4", 128, 512)["codes"], ox["codes"])
    yr, bd = O.gemm_ref(ox, ow, "mxfp4")
    _check(host_f32(y), yr, bd)


SHAPES = [(128, 128, 256), (200, 300, 512), (1, 256, 4096), (16, 512, 320), (257, 129, 576), (384, 1024, 1024)]


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("mnk", SHAPES)
def test_gemm_shapes(mnk, fmt):
    M, N, K = mnk
    g = np.random.default_rng(M * 31 + N * 7 + K)
    from workloads import bf16_bits
    a = bf16_bits(g.standard_normal((M, K)).astype(np.float32))
    b = bf16_bits((g.standard_normal((N, K)) * 0.02).astype(np.float32))
    qa, qb = _gpu_quant(dev_bf16(a), fmt), _gpu_quant(dev_bf16(b), fmt)
    y32 = F.fp4_gemm(qa.codes, qa.scales, qb.codes, qb.scales, fmt=fmt, a_tensor_scale=qa.tensor_scale,
                     b_tensor_scale=qb.tensor_scale, out_dtype="f32")
    y16 = F.fp4_gemm(qa.codes, qa.scales, qb.codes, qb.scales, fmt=fmt, a_tensor_scale=qa.tensor_scale,
                     b_tensor_scale=qb.tensor_scale, out_dtype="bf16")
    yr, bd = O.gemm_ref(_as_oracle(qa, fmt, M, K), _as_oracle(qb, fmt, N, K), fmt)
    got = host_f32(y32)
    _check(got, yr, bd)
    _bf16_ulp_check(y16, got)
    F.fp4_check_device_errors()


SMALL_M = [1, 2, 3, 4, 5, 16, 17, 32, 33, 64, 65, 127, 128]
SMALL_NK = [(128, 4096), (300, 320), (4100, 1024)]


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("nk", SMALL_NK)
@pytest.mark.parametrize("M", SMALL_M)
def test_gemm_small_m_weight_streaming(M, nk, fmt):
    """At most 128 activation rows: the weights stream through the MMA's M dimension in 128-row
    tiles with the activations as its N (16, 32, 64 or 128 columns), k-tiles split over a cluster.
    Ragged M inside each activation tile width, a ragged last weight tile (N = 300, 4100), a k-tail
    (K = 320: one 256-wide k-tile and one of 64), a single weight tile split eight ways (N = 128);
    fp32 output against the fp64 oracle, bf16 within one ulp of it, and a strided output."""
    N, K = nk
    g = np.random.default_rng(M * 131 + N + K)
    from workloads import bf16_bits
    a = bf16_bits(g.standard_normal((M, K)).astype(np.float32))
    b = bf16_bits((g.standard_normal((N, K)) * 0.02).astype(np.float32))
    qa, qb = _gpu_quant(dev_bf16(a), fmt), _gpu_quant(dev_bf16(b), fmt)
    kw = dict(fmt=fmt, a_tensor_scale=qa.tensor_scale, b_tensor_scale=qb.tensor_scale)
    y32 = F.fp4_gemm(qa.codes, qa.scales, qb.codes, qb.scales, out_dtype="f32", **kw)
    y16 = F.fp4_gemm(qa.codes, qa.scales, qb.codes, qb.scales, out_dtype="bf16", **kw)
    big = torch.full((M, N + 36), 7.0, dtype=torch.float32, device="cuda")
    F.fp4_gemm(qa.codes, qa.scales, qb.codes, qb.scales, out_dtype="f32", out=big[:, :N], **kw)
    yr, bd = O.gemm_ref(_as_oracle(qa, fmt, M, K), _as_oracle(qb, fmt, N, K), fmt)
    got = host_f32(y32)
    _check(got, yr, bd)
    _bf16_ulp_check(y16, got)
    out = host_f32(big)
    np.testing.assert_array_equal(out[:, :N].view(np.uint32), got.view(np.uint32))
    assert np.all(out[:, N:] == 7.0)            # nothing written past N
    F.fp4_check_device_errors()


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("M, N, K", [(1, 4096, 4096), (1, 11008, 4096), (1, 4096, 11008), (1, 1000, 11008),
                                     (1, 77, 64), (1, 1, 128)])
def test_gemm_cuda_core_rows(M, N, K, fmt):
    """One activation row runs on the CUDA cores (exact f16 block sums, fp32 across blocks): the
    Llama-7B decode shapes, a ragged N, the shortest K, a single output; a heavy-tailed activation
    row with a zero block; fp32 against the fp64 oracle (sampled columns for the large N), bf16
    within one ulp, and a strided output.  N = 1000 x K = 11008 (weights for every SM, too few rows
    to give each SM two CTAs of 16) stages each SM's rows whole in shared memory; the others stream
    rows through the warps' registers."""
    g = np.random.default_rng(M * 7 + N + K)
    from workloads import bf16_bits
    a = mixed_input(M, K, M + K, fmt)
    b = bf16_bits((g.standard_t(4, (N, K)) * 0.02).astype(np.float32))
    qa, qb = _gpu_quant(dev_bf16(a), fmt), _gpu_quant(dev_bf16(b), fmt)
    kw = dict(fmt=fmt, a_tensor_scale=qa.tensor_scale, b_tensor_scale=qb.tensor_scale)
    y32 = F.fp4_gemm(qa.codes, qa.scales, qb.codes, qb.scales, out_dtype="f32", **kw)
    y16 = F.fp4_gemm(qa.codes, qa.scales, qb.codes, qb.scales, out_dtype="bf16", **kw)
    big = torch.full((M, N + 20), 7.0, dtype=torch.float32, device="cuda")
    F.fp4_gemm(qa.codes, qa.scales, qb.codes, qb.scales, out_dtype="f32", out=big[:, :N], **kw)
    rows = np.arange(N) if N <= 1000 else np.sort(np.random.default_rng(1).choice(N, 1000, replace=False))
    yr, bd = O.gemm_ref_cols(_as_oracle(qa, fmt, M, K), _as_oracle(qb, fmt, N, K), fmt, rows)
    got = host_f32(y32)
    _check(got[:, rows], yr, bd)
    _bf16_ulp_check(y16, got)
    out = host_f32(big)
    np.testing.assert_array_equal(out[:, :N].view(np.uint32), got.view(np.uint32))
    assert np.all(out[:, N:] == 7.0)
    F.fp4_check_device_errors()


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_pair_tiles_ragged_edges(fmt):
    """2400 x 1900 x 2048: enough 256 x 256 tiles for the SM-pair kernel, with the last row tile's
    second 128-row half and the last column tile's second 128-row scale block outside the operands
    (their boxes read the tensor map's zero fill)."""
    M, N, K = 2400, 1900, 2048
    g = np.random.default_rng(77)
    from workloads import bf16_bits
    a = bf16_bits(g.standard_normal((M, K)).astype(np.float32))
    b = bf16_bits((g.standard_normal((N, K)) * 0.02).astype(np.float32))
    qa, qb = _gpu_quant(dev_bf16(a), fmt), _gpu_quant(dev_bf16(b), fmt)
    y32 = F.fp4_gemm(qa.codes, qa.scales, qb.codes, qb.scales, fmt=fmt, a_tensor_scale=qa.tensor_scale,
                     b_tensor_scale=qb.tensor_scale, out_dtype="f32")
    yr, bd = O.gemm_ref(_as_oracle(qa, fmt, M, K), _as_oracle(qb, fmt, N, K), fmt)
    _check(host_f32(y32), yr, bd)
    F.fp4_check_device_errors()


def test_gemm_strided_output():
    M, N, K = 64, 96, 256
    g = np.random.default_rng(1)
    from workloads import bf16_bits
    a = bf16_bits(g.standard_normal((M, K)).astype(np.float32))
    b = bf16_bits(g.standard_normal((N, K)).astype(np.float32))
    qa, qb = _gpu_quant(dev_bf16(a), "mxfp4"), _gpu_quant(dev_bf16(b), "mxfp4")
    big = torch.full((M, 128), 7.0, dtype=torch.float32, device="cuda")
    F.fp4_gemm(qa.codes, qa.scales, qb.codes, qb.scales, fmt="mxfp4", out_dtype="f32", out=big[:, :N])
    yr, bd = O.gemm_ref(_as_oracle(qa, "mxfp4", M, K), _as_oracle(qb, "mxfp4", N, K), "mxfp4")
    out = host_f32(big)
    _check(out[:, :N], yr, bd)
    assert np.all(out[:, N:] == 7.0)          # nothing written past N


@pytest.mark.parametrize("had", [16, 128])
def test_full_size_hadamard_mxfp4_8192x11008x4096(had):
    """X[8192,4096] N(0,1) with 41 channels x50, rotated online; W[11008,4096] N(0,0.02) rotated
    and quantized offline; 64 sampled rows and 64 sampled columns of Y checked (fp32 run), bf16 run
    against the fp32 run."""
    xb = hadamard_acts(8192, 4096, seed=2)
    wb = hadamard_weights(11008, 4096, seed=2)
    qw = F.fp4_hadamard_quantize(dev_bf16(wb), had, fmt="mxfp4", sf_layout="mma")   # offline weights
    qx = F.fp4_hadamard_quantize(dev_bf16(xb), had, fmt="mxfp4", sf_layout="mma")
    y16 = F.fp4_gemm(qx.codes, qx.scales, qw.codes, qw.scales, fmt="mxfp4", out_dtype="bf16")
    y32 = F.fp4_gemm(qx.codes, qx.scales, qw.codes, qw.scales, fmt="mxfp4", out_dtype="f32")
    oa, ob = _as_oracle(qx, "mxfp4", 8192, 4096), _as_oracle(qw, "mxfp4", 11008, 4096)
    g = np.random.default_rng(had)
    rows = np.sort(g.choice(8192, 64, replace=False))
    cols = np.sort(g.choice(11008, 64, replace=False))
    yr, bd = O.gemm_ref_rows(oa, ob, "mxfp4", rows)
    full32 = y32[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    _check(full32, yr, bd)
    yc, bc = O.gemm_ref_cols(oa, ob, "mxfp4", cols)
    _check(y32[:, torch.from_numpy(cols).cuda()].float().cpu().numpy(), yc, bc)
    _bf16_ulp_check(y16[torch.from_numpy(rows).cuda()], full32)
    F.fp4_check_device_errors()


@pytest.mark.parametrize("layer", ["qkv", "fc1", "fc2"])
def test_vit_fwd_dgrad_wgrad_full_size(layer):
    """ViT-B/16 linear (qkv 768->2304, fc1 768->3072, fc2 3072->768), M = 50432: forward (RTN), dgrad and wgrad with SR-quantized dY,
    each operand quantized along its own contraction axis (axis 0 = transposed blocks)."""
    xb, wb, dyb = vit_layer(layer)
    M, K = xb.shape
    N = wb.shape[0]
    x, w, dy = dev_bf16(xb), dev_bf16(wb), dev_bf16(dyb)
    g = np.random.default_rng(3)
    # forward Y = X W^T, contraction K
    qx, qw = _gpu_quant(x, "mxfp4"), _gpu_quant(w, "mxfp4")
    y = F.fp4_gemm(qx.codes, qx.scales, qw.codes, qw.scales, fmt="mxfp4", out_dtype="f32")
    rows = np.sort(g.choice(M, 64, replace=False))
    yr, bd = O.gemm_ref_rows(_as_oracle(qx, "mxfp4", M, K), _as_oracle(qw, "mxfp4", N, K), "mxfp4", rows)
    _check(y[torch.from_numpy(rows).cuda()].cpu().numpy(), yr, bd)
    # dgrad dX = dY W, contraction N: dY along N (SR, seed 3), W along N (axis 0, RTN)
    qdy = _gpu_quant(dy, "mxfp4", axis=1, rnd="sr", seed=3)
    qwt = _gpu_quant(w, "mxfp4", axis=0)
    dx = F.fp4_gemm(qdy.codes, qdy.scales, qwt.codes, qwt.scales, fmt="mxfp4", out_dtype="f32")
    yr, bd = O.gemm_ref_rows(_as_oracle(qdy, "mxfp4", M, N), _as_oracle(qwt, "mxfp4", K, N), "mxfp4", rows)
    _check(dx[torch.from_numpy(rows).cuda()].cpu().numpy(), yr, bd)
    # wgrad dW = dY^T X, contraction M: dY along M (axis 0, SR, seed 4), X along M (axis 0, RTN)
    qdyt = _gpu_quant(dy, "mxfp4", axis=0, rnd="sr", seed=4)
    qxt = _gpu_quant(x, "mxfp4", axis=0)
    dw = F.fp4_gemm(qdyt.codes, qdyt.scales, qxt.codes, qxt.scales, fmt="mxfp4", out_dtype="f32")
    wrows = np.sort(g.choice(N, 32, replace=False))
    yr, bd = O.gemm_ref_rows(_as_oracle(qdyt, "mxfp4", N, M), _as_oracle(qxt, "mxfp4", K, M), "mxfp4", wrows)
    _check(dw[torch.from_numpy(wrows).cuda()].cpu().numpy(), yr, bd)
    # the SR operands themselves: sampled output rows against the oracle with global Philox indices
    dy32 = bf16_to_f32(dyb)
    for c in np.sort(g.choice(N, 8, replace=False)):
        ref = O.quantize_values(dy32[:, c:c + 1], fmt="mxfp4", axis=0, rnd="sr", seed=4, idx_base=int(c), idx_cols=N)
        np.testing.assert_array_equal(host_u8(qdyt.codes[c:c + 1]), ref["codes"])
        np.testing.assert_array_equal(
            O.sf_from_mma(host_u8(qdyt.scales), N, M // 32)[c:c + 1], ref["scales"])
    F.fp4_check_device_errors()


@pytest.mark.parametrize("kn", [(4096, 4096), (4096, 11008), (11008, 4096)])
def test_llama_nvfp4_sweep(kn):
    """Llama-7B shapes, NVFP4: X[:M] (0.5% channels x20, generated at 16384 rows) amax + quantize
    along K, W quantized once; M = 1, 16, 128, 1024, 4096, 16384.  Per M: the tensor scale equals
    the oracle's, sampled rows of codes and scales are bit-exact, and sampled output rows (all
    rows for M <= 128) and columns (M <= 4096) of the fp32 GEMM meet the bound."""
    K, N = kn
    xb = llama_acts(K, 16384, seed=4)
    wb = llama_weights(K, N, seed=4)
    x, w = dev_bf16(xb), dev_bf16(wb)
    qw = _gpu_quant(w, "nvfp4")
    ob = _as_oracle(qw, "nvfp4", N, K)
    w32 = bf16_to_f32(wb)
    assert ob["tensor_scale"] == O.nv_tensor_scale(w32)
    g = np.random.default_rng(K + N)
    wr = np.sort(g.choice(N, 16, replace=False))
    ref = O.quantize_values(w32[wr], fmt="nvfp4", tensor_scale=ob["tensor_scale"])
    np.testing.assert_array_equal(ob["codes"][wr], ref["codes"])
    np.testing.assert_array_equal(ob["scales"][wr], ref["scales"])
    x32 = bf16_to_f32(xb)
    for M in (1, 16, 128, 1024, 4096, 16384):
        qx = _gpu_quant(x[:M], "nvfp4")
        oa = _as_oracle(qx, "nvfp4", M, K)
        assert oa["tensor_scale"] == O.nv_tensor_scale(x32[:M]), M
        rows = np.arange(M) if M <= 128 else np.sort(g.choice(M, 32, replace=False))
        sample = rows[:16]
        ref = O.quantize_values(x32[sample], fmt="nvfp4", tensor_scale=oa["tensor_scale"])
        np.testing.assert_array_equal(oa["codes"][sample], ref["codes"])
        np.testing.assert_array_equal(oa["scales"][sample], ref["scales"])
        y = F.fp4_gemm(qx.codes, qx.scales, qw.codes, qw.scales, fmt="nvfp4", a_tensor_scale=qx.tensor_scale,
                       b_tensor_scale=qw.tensor_scale, out_dtype="f32")
        yr, bd = O.gemm_ref_rows(oa, ob, "nvfp4", rows)
        _check(y[torch.from_numpy(rows).cuda()].cpu().numpy(), yr, bd)
        if M <= 4096:
            cols = np.sort(g.choice(N, 16, replace=False))
            yc, bc = O.gemm_ref_cols(oa, ob, "nvfp4", cols)
            _check(y[:, torch.from_numpy(cols).cuda()].cpu().numpy(), yc, bc)
        y16 = F.fp4_gemm(qx.codes, qx.scales, qw.codes, qw.scales, fmt="nvfp4", a_tensor_scale=qx.tensor_scale,
                         b_tensor_scale=qw.tensor_scale, out_dtype="bf16")
        _bf16_ulp_check(y16[torch.from_numpy(rows).cuda()], y[torch.from_numpy(rows).cuda()].cpu().numpy())
    F.fp4_check_device_errors()
