"""GPU parity of the GEMM with the fused output quantizer (fp4_gemm_quantize): the next layer's FP4
codes and scales straight from the accumulators.

Exact cases: operands built on the host from seeded codes with scales drawn from a few powers of
two (MXFP4 bytes 126..128; NVFP4 E4M3 0.5, 1, 2 with unit tensor scales) and K <= 2048, so every
product and partial sum is exact in fp32 and the accumulation order cannot change Y: the fused
codes and scales must equal the oracle's quantization of its fp64 product bit for bit.  A realistic
case (quantized N(0,1) activations and N(0,0.02) weights) is checked against the oracle's product
within the GEMM's error bound: codes differ only by one grid step, scales by one, where Y sits on a
rounding boundary."""
import numpy as np
import pytest
import torch

import oracle as O
import microscaling_fp4_quantization_mxfp4_b200 as F
from gpu_utils import dev_bf16, host_f32, host_u8
from workloads import bf16_to_f32, normal_bf16

pytestmark = pytest.mark.gpu


def _operand(rows, k, fmt, seed):
    """Seeded FP4 operand: random codes, scale bytes from a small set of powers of two."""
    g = np.random.default_rng(seed)
    codes = g.integers(0, 256, size=(rows, k // 2), dtype=np.uint8)
    if fmt == "mxfp4":
        scales = g.integers(126, 129, size=(rows, k // 32)).astype(np.uint8)
    else:
        scales = g.choice(np.array([48, 56, 64], dtype=np.uint8), size=(rows, k // 16))
    return {"codes": codes, "scales": scales, "tensor_scale": np.float32(1.0) if fmt == "nvfp4" else None}


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _run(A, B, fmt, out_fmt, rnd, seed, sf, ts=None):
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    ts_dev = None if ts is None else torch.tensor([ts], dtype=torch.float32, device="cuda")
    return F.fp4_gemm_quantize(_dev(A["codes"]), _dev(O.sf_to_mma(A["scales"])), _dev(B["codes"]),
                               _dev(O.sf_to_mma(B["scales"])), fmt=fmt,
                               a_tensor_scale=one if fmt == "nvfp4" else None,
                               b_tensor_scale=one if fmt == "nvfp4" else None, out_fmt=out_fmt, rnd=rnd, seed=seed,
                               out_tensor_scale=ts_dev, out_sf_layout=sf)


def _check_exact(q, ref, sf, M, N, bs):
    np.testing.assert_array_equal(host_u8(q.codes), ref["codes"])
    got = host_u8(q.scales)
    if sf == "mma":
        np.testing.assert_array_equal(O.sf_from_mma(got, M, N // bs), ref["scales"])
        np.testing.assert_array_equal(got, O.sf_to_mma(ref["scales"]))
    else:
        np.testing.assert_array_equal(got, ref["scales"])


@pytest.mark.parametrize("fmt, out_fmt, rnd, sf, mnk", [
    ("mxfp4", "mxfp4", "rtn", "mma", (300, 352, 1024)),          # single-SM 128x256 tiles, ragged M and N
    ("mxfp4", "mxfp4", "sr", "rowmajor", (300, 160, 1024)),      # 128x128 tiles
    ("nvfp4", "nvfp4", "rtn", "mma", (256, 288, 512)),
    ("nvfp4", "nvfp4", "sr", "mma", (130, 256, 1024)),
    ("mxfp4", "mxfp4_gs", "rtn", "rowmajor", (200, 256, 768)),
    ("nvfp4", "mxfp4", "sr", "mma", (128, 512, 256)),
    ("mxfp4", "nvfp4", "rtn", "rowmajor", (2048, 2560, 2048)),    # SM-pair 256x256 tiles
    ("nvfp4", "mxfp4", "sr", "mma", (2048, 2560, 2048)),
])
def test_fused_quantize_exact(fmt, out_fmt, rnd, sf, mnk):
    M, N, K = mnk
    A, B = _operand(M, K, fmt, 7 + M), _operand(N, K, fmt, 11 + N)
    y64, _ = O.gemm_ref(A, B, fmt)
    y32 = y64.astype(np.float32)
    assert np.array_equal(y32.astype(np.float64), y64)               # exact in fp32 by construction
    ts = None
    if out_fmt == "nvfp4":
        ts = np.float32(O.nv_tensor_scale(y32) * np.float32(1.25))      # a caller's (stale) scale
    q = _run(A, B, fmt, out_fmt, rnd, 99, sf, ts)
    ref = O.quantize_values(y32, fmt=out_fmt, rnd=rnd, seed=99, tensor_scale=ts)
    _check_exact(q, ref, sf, M, N, 32 if out_fmt.startswith("mx") else 16)
    F.fp4_check_device_errors()


def test_fused_quantize_feeds_the_next_gemm():
    """Layer 1's fused output is layer 2's A operand: the second GEMM on it equals the oracle's."""
    M, N, K, N2 = 256, 512, 1024, 384
    A, B = _operand(M, K, "mxfp4", 1), _operand(N, K, "mxfp4", 2)
    C = _operand(N2, N, "mxfp4", 3)
    q = _run(A, B, "mxfp4", "mxfp4", "rtn", 0, "mma")
    y2 = F.fp4_gemm(q.codes, q.scales, _dev(C["codes"]), _dev(O.sf_to_mma(C["scales"])), fmt="mxfp4", out_dtype="f32")
    y64, _ = O.gemm_ref(A, B, "mxfp4")
    mid = O.quantize_values(y64.astype(np.float32), fmt="mxfp4")
    want, bound = O.gemm_ref(mid, C, "mxfp4")
    assert np.all(np.abs(host_f32(y2) - want) <= 1e-5 * bound)
    F.fp4_check_device_errors()


def test_fused_quantize_realistic_operands():
    """Quantized N(0,1) activations x N(0,0.02) weights, 1024 x 1024 x 2048 (fp32 accumulation is
    not exact here): against the oracle's quantization of its fp64 product, at most 1e-3 of codes
    differ, each by one grid step, and every scale byte is within one."""
    M, N, K = 1024, 1024, 2048
    xb = normal_bf16((M, K), 1.0, 50, 0)
    wb = normal_bf16((N, K), 0.02, 50, 1)
    A, B = O.quantize(xb, fmt="nvfp4"), O.quantize(wb, fmt="nvfp4")
    ta = torch.tensor([A["tensor_scale"]], dtype=torch.float32, device="cuda")
    tb = torch.tensor([B["tensor_scale"]], dtype=torch.float32, device="cuda")
    q = F.fp4_gemm_quantize(_dev(A["codes"]), _dev(O.sf_to_mma(A["scales"])), _dev(B["codes"]),
                            _dev(O.sf_to_mma(B["scales"])), fmt="nvfp4", a_tensor_scale=ta, b_tensor_scale=tb,
                            out_fmt="mxfp4", rnd="rtn", out_sf_layout="rowmajor")
    y64, _ = O.gemm_ref(A, B, "nvfp4")
    ref = O.quantize_values(y64.astype(np.float32), fmt="mxfp4")
    gs, rs = host_u8(q.scales).astype(np.int64), ref["scales"].astype(np.int64)
    assert np.all(np.abs(gs - rs) <= 1) and (gs != rs).mean() <= 1e-2
    gc = O.unpack_nibbles(host_u8(q.codes)).astype(np.int64)
    rc = O.unpack_nibbles(ref["codes"]).astype(np.int64)
    same_scale = np.repeat(gs == rs, 32, axis=1)
    gpos = np.where(gc & 8, -(gc & 7), gc & 7)
    rpos = np.where(rc & 8, -(rc & 7), rc & 7)
    diff = (gpos != rpos) & same_scale
    assert diff.mean() <= 1e-3
    assert np.all(np.abs(gpos - rpos)[same_scale] <= 1)
    F.fp4_check_device_errors()
