"""Pins for the oracle's block-Hadamard rotation (CPU only)."""
import numpy as np
import pytest
import scipy.linalg

import oracle as O


@pytest.mark.parametrize("n", [1, 2, 4, 16, 32, 64, 128])
def test_sylvester_matches_scipy(n):
    np.testing.assert_array_equal(O.sylvester(n), scipy.linalg.hadamard(n))


@pytest.mark.parametrize("n", [16, 32, 64, 128])
def test_orthogonality_and_popcount_form(n):
    h = O.sylvester(n)
    np.testing.assert_array_equal(h @ h.T, n * np.eye(n))
    i, j = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
    pc = np.vectorize(lambda v: bin(v).count("1"))(i & j)
    np.testing.assert_array_equal(h, (-1.0) ** pc)


@pytest.mark.parametrize("b", [16, 32, 64, 128])
def test_block_rotation_norm_involution_blockdiag(b):
    rng = np.random.default_rng(b)
    x = rng.standard_normal((8, 512))
    y = O.block_hadamard(x, b)
    # each block keeps its norm
    np.testing.assert_allclose(np.linalg.norm(y.reshape(8, -1, b), axis=2),
                               np.linalg.norm(x.reshape(8, -1, b), axis=2), rtol=1e-12)
    # the normalised Sylvester matrix is symmetric orthogonal: applying it twice is the identity
    np.testing.assert_allclose(O.block_hadamard(y, b), x, rtol=0, atol=1e-12)
    # equals multiplication by the block-diagonal matrix
    bd = scipy.linalg.block_diag(*([scipy.linalg.hadamard(b) / np.sqrt(b)] * (512 // b)))
    np.testing.assert_allclose(y, x @ bd, rtol=0, atol=1e-12)
    # axis 0 is axis 1 of the transpose
    np.testing.assert_allclose(O.block_hadamard(x.T, b, axis=0), y.T, rtol=0, atol=0)


def test_rotation_preserves_products_with_rotated_weights():
    # X' W'^T = X W^T: the rotation fused into the weights cancels in the GEMM
    rng = np.random.default_rng(0)
    x = rng.standard_normal((4, 256))
    w = rng.standard_normal((3, 256))
    np.testing.assert_allclose(O.block_hadamard(x, 64) @ O.block_hadamard(w, 64).T, x @ w.T, atol=1e-10)


def test_quantize_with_rotation_rounds_rotated_values_to_fp32():
    from workloads import bf16_bits, bf16_to_f32
    rng = np.random.default_rng(6)
    xb = bf16_bits(rng.standard_normal((4, 128)).astype(np.float32))
    r = O.quantize(xb, fmt="mxfp4", had_block=128)
    want = O.block_hadamard(bf16_to_f32(xb).astype(np.float64), 128).astype(np.float32)
    np.testing.assert_array_equal(r["rotated"], want)
