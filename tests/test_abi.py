"""The C ABI library without a GPU: it builds, loads, exports every function that
include/*.h declares, and rejects invalid arguments before any CUDA call."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from microscaling_fp4_quantization_mxfp4_b200 import build, _lib
    build.build()
    return _lib.load()


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b(fp4_[a-z0-9_]+)\s*\(", src))
    return names


def test_header_declares_the_boundary():
    assert {"fp4_quantize", "fp4_dequantize", "fp4_hadamard_quantize", "fp4_gemm"} <= _declared()


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in sorted(_declared()) if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_prototypes_cover_the_header():
    from microscaling_fp4_quantization_mxfp4_b200 import _lib
    assert _declared() == set(_lib.PROTOTYPES)


def test_size_helpers(lib):
    assert lib.fp4_codes_bytes(4096, 4096) == 4096 * 2048
    assert lib.fp4_scales_bytes(4096, 4096, 16, 1, 0) == 4096 * 256
    assert lib.fp4_scales_bytes(130, 64, 32, 1, 1) == 256 * 4          # rows padded to 128, groups to 4
    assert lib.fp4_scales_bytes(64, 96, 32, 0, 0) == 96 * 2             # axis 0: [cols, rows/block]
    assert lib.fp4_scales_bytes(64, 100, 32, 1, 0) == 0                 # not a multiple of the block


def test_status_strings(lib):
    for code in range(0, -7, -1):
        assert lib.fp4_status_string(code)
    assert lib.fp4_status_string(-3) == b"misaligned pointer or leading dimension"


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails validation first


@pytest.mark.parametrize("args, status", [
    # x null
    ((None, 4, 64, 64, 0, 32, 1, 0, 0, None, None, FAKE, FAKE, 0, None), -1),
    # unsupported (format, block)
    ((FAKE, 4, 64, 64, 0, 16, 1, 0, 0, None, None, FAKE, FAKE, 0, None), -4),
    # cols not a multiple of 8
    ((FAKE, 4, 60, 64, 0, 32, 1, 0, 0, None, None, FAKE, FAKE, 0, None), -2),
    # misaligned x
    ((FAKE + 2, 4, 64, 64, 0, 32, 1, 0, 0, None, None, FAKE, FAKE, 0, None), -3),
    # axis-1 length not a multiple of the block
    ((FAKE, 4, 40, 40, 0, 32, 1, 0, 0, None, None, FAKE, FAKE, 0, None), -2),
    # NVFP4 without tensor_scale_out
    ((FAKE, 4, 64, 64, 1, 16, 1, 0, 0, None, None, FAKE, FAKE, 0, None), -1),
    # bad axis / rounding / layout
    ((FAKE, 4, 64, 64, 0, 32, 2, 0, 0, None, None, FAKE, FAKE, 0, None), -1),
    ((FAKE, 4, 64, 64, 0, 32, 1, 5, 0, None, None, FAKE, FAKE, 0, None), -1),
    ((FAKE, 4, 64, 64, 0, 32, 1, 0, 0, None, None, FAKE, FAKE, 7, None), -1),
])
def test_quantize_rejects_before_launch(lib, args, status):
    assert lib.fp4_quantize(*args) == status


def test_other_entry_points_reject_before_launch(lib):
    assert lib.fp4_hadamard_quantize(FAKE, 4, 64, 64, 0, 32, 1, 0, 0, None, None, FAKE, FAKE, 0, 8, None, None) == -1
    assert lib.fp4_hadamard_quantize(FAKE, 64, 64, 64, 0, 32, 0, 0, 0, None, None, FAKE, FAKE, 0, 32, None, None) == -4
    assert lib.fp4_hadamard_quantize(FAKE, 4, 96, 96, 0, 32, 1, 0, 0, None, None, FAKE, FAKE, 0, 64, None, None) == -2
    assert lib.fp4_dequantize(FAKE, FAKE, None, 4, 64, 1, 16, 0, FAKE, 0, None) == -1     # NV needs s_t
    assert lib.fp4_dequantize(FAKE, FAKE, None, 4, 64, 0, 32, 0, FAKE, 9, None) == -1
    assert lib.fp4_gemm(FAKE, FAKE, None, FAKE, FAKE, None, 4, 4, 96, 0, 32, FAKE, 4, 0, None) == -2   # K % 64
    assert lib.fp4_gemm(FAKE, FAKE, None, FAKE, FAKE, None, 4, 4, 64, 1, 16, FAKE, 4, 0, None) == -1   # NV scales
    assert lib.fp4_gemm(FAKE, FAKE, None, FAKE, FAKE, None, 4, 8, 64, 0, 32, FAKE, 4, 0, None) == -1   # ldy < N
    assert lib.fp4_gemm(FAKE + 8, FAKE, None, FAKE, FAKE, None, 4, 4, 64, 0, 32, FAKE, 4, 0, None) == -3
    assert lib.fp4_amax(None, 4, 64, 64, FAKE, None) == -1
    assert lib.fp4_amax_noalloc(FAKE, 8192, 8200, 8200, FAKE, None) == -2                # beyond its scratch
    assert lib.fp4_nv_tensor_scale(None, FAKE, None) == -1
    # fp4_quantize_2d: rows not a multiple of the tile, half of the transposed pair, NV without s_t out
    assert lib.fp4_quantize_2d(FAKE, 40, 64, 64, 0, 32, 0, 0, None, None, FAKE, FAKE, None, None, 0, None) == -2
    assert lib.fp4_quantize_2d(FAKE, 64, 64, 64, 0, 32, 0, 0, None, None, FAKE, FAKE, FAKE, None, 0, None) == -1
    assert lib.fp4_quantize_2d(FAKE, 64, 64, 64, 1, 16, 0, 0, None, None, FAKE, FAKE, None, None, 0, None) == -1
    assert lib.fp4_quantize_2d(FAKE, 64, 64, 64, 0, 32, 0, 0, None, None, FAKE + 4, FAKE, None, None, 0, None) == -3
    # fp4_quantize_shard: negative first row, axis-0 shard not starting on a block, then fp4_quantize's checks
    assert lib.fp4_quantize_shard(FAKE, 4, 64, 64, -16, 0, 32, 1, 0, 0, None, None, FAKE, FAKE, 0, None) == -1
    assert lib.fp4_quantize_shard(FAKE, 64, 64, 64, 16, 0, 32, 0, 0, 0, None, None, FAKE, FAKE, 0, None) == -2
    assert lib.fp4_quantize_shard(FAKE, 4, 64, 64, 8, 0, 16, 1, 0, 0, None, None, FAKE, FAKE, 0, None) == -4
    assert lib.fp4_quantize_shard(FAKE + 2, 4, 64, 64, 8, 0, 32, 1, 0, 0, None, None, FAKE, FAKE, 0, None) == -3
    # four-over-six NVFP4 (fmt 2): block 16 only, needs s_t out, no Hadamard, quantizer entry points only
    assert lib.fp4_quantize(FAKE, 4, 64, 64, 2, 32, 1, 0, 0, None, None, FAKE, FAKE, 0, None) == -4
    assert lib.fp4_quantize(FAKE, 4, 64, 64, 2, 16, 1, 0, 0, None, None, FAKE, FAKE, 0, None) == -1
    assert lib.fp4_hadamard_quantize(FAKE, 4, 64, 64, 2, 16, 1, 0, 0, None, FAKE, FAKE, FAKE, 0, 16, None, None) == -4
    assert lib.fp4_dequantize(FAKE, FAKE, FAKE, 4, 64, 2, 16, 0, FAKE, 0, None) == -1
    assert lib.fp4_gemm(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 4, 64, 2, 16, FAKE, 4, 0, None) == -1
    # MXFP4 with the fitted clip threshold (fmt 3): block 32 only, quantizer entry points only
    assert lib.fp4_quantize(FAKE, 4, 64, 64, 3, 16, 1, 0, 0, None, None, FAKE, FAKE, 0, None) == -4
    assert lib.fp4_quantize_2d(FAKE, 64, 64, 64, 3, 32, 0, 0, None, None, FAKE, FAKE, None, None, 0, None) == -1
    # fp4_quantize_mse: NVFP4 block 16 only, iters in [0, 8], s_t out required, cols % 16
    assert lib.fp4_quantize_mse(FAKE, 4, 64, 64, 0, 32, 0, 0, 1, FAKE, FAKE, FAKE, 0, None) == -4
    assert lib.fp4_quantize_mse(FAKE, 4, 64, 64, 1, 16, 0, 0, 9, FAKE, FAKE, FAKE, 0, None) == -1
    assert lib.fp4_quantize_mse(FAKE, 4, 64, 64, 1, 16, 0, 0, 1, None, FAKE, FAKE, 0, None) == -1
    assert lib.fp4_quantize_mse(FAKE, 4, 40, 40, 1, 16, 0, 0, 1, FAKE, FAKE, FAKE, 0, None) == -2
    assert lib.fp4_quantize_mse(FAKE, 4, 64, 64, 1, 16, 2, 0, 1, FAKE, FAKE, FAKE, 0, None) == -1
    # fp4_gemm_quantize: N % 32, NV output needs a tensor scale, output (format, block) pairs
    assert lib.fp4_gemm_quantize(FAKE, FAKE, None, FAKE, FAKE, None, 4, 48, 64, 0, 32, 0, 32, 0, 0, None, FAKE, FAKE,
                                 1, None) == -2
    assert lib.fp4_gemm_quantize(FAKE, FAKE, None, FAKE, FAKE, None, 4, 64, 64, 0, 32, 1, 16, 0, 0, None, FAKE, FAKE,
                                 1, None) == -1
    assert lib.fp4_gemm_quantize(FAKE, FAKE, None, FAKE, FAKE, None, 4, 64, 64, 0, 32, 0, 16, 0, 0, None, FAKE, FAKE,
                                 1, None) == -4
    assert lib.fp4_gemm_quantize(FAKE, FAKE, None, FAKE, FAKE, None, 4, 64, 64, 0, 32, 2, 16, 0, 0, FAKE, FAKE, FAKE,
                                 1, None) == -1
    assert lib.fp4_gemm_quantize(FAKE, FAKE, None, FAKE, FAKE, None, 4, 64, 64, 0, 32, 0, 32, 0, 0, None, FAKE + 8,
                                 FAKE, 1, None) == -3
    # fp4_quantize_dequantize: output required, dtype, no four-over-six, aligned output
    assert lib.fp4_quantize_dequantize(FAKE, 4, 64, 64, 0, 32, 0, 0, None, None, FAKE, FAKE, 0, None, 0, None) == -1
    assert lib.fp4_quantize_dequantize(FAKE, 4, 64, 64, 0, 32, 0, 0, None, None, FAKE, FAKE, 0, FAKE, 5, None) == -1
    assert lib.fp4_quantize_dequantize(FAKE, 4, 64, 64, 2, 16, 0, 0, None, FAKE, FAKE, FAKE, 0, FAKE, 0, None) == -4
    assert lib.fp4_quantize_dequantize(FAKE, 4, 64, 64, 0, 32, 0, 0, None, None, FAKE, FAKE, 0, FAKE + 4, 0,
                                       None) == -3


@pytest.mark.parametrize("rows, cols", [(0, 64), (64, 0), (0, 0), (-1, 64)])
def test_empty_and_negative_shapes_rejected(lib, rows, cols):
    """Zero-sized (and negative) tensors are argument errors at every entry point, returned before
    any CUDA call; the size helpers report 0 bytes for them."""
    assert lib.fp4_quantize(FAKE, rows, cols, max(cols, 1), 0, 32, 1, 0, 0, None, None, FAKE, FAKE, 0, None) == -1
    assert lib.fp4_quantize(FAKE, rows, cols, max(cols, 1), 1, 16, 1, 0, 0, None, FAKE, FAKE, FAKE, 0, None) == -1
    assert lib.fp4_hadamard_quantize(FAKE, rows, cols, max(cols, 1), 0, 32, 1, 0, 0, None, None, FAKE, FAKE, 0, 32,
                                     None, None) == -1
    assert lib.fp4_quantize_dequantize(FAKE, rows, cols, max(cols, 1), 0, 32, 0, 0, None, None, FAKE, FAKE, 0, FAKE,
                                       0, None) == -1
    assert lib.fp4_quantize_2d(FAKE, rows, cols, max(cols, 1), 0, 32, 0, 0, None, None, FAKE, FAKE, None, None, 0,
                               None) == -1
    assert lib.fp4_quantize_mse(FAKE, rows, cols, max(cols, 1), 1, 16, 0, 0, 1, FAKE, FAKE, FAKE, 0, None) == -1
    assert lib.fp4_dequantize(FAKE, FAKE, None, rows, cols, 0, 32, 0, FAKE, 0, None) == -1
    assert lib.fp4_amax(FAKE, rows, cols, max(cols, 1), FAKE, None) == -1
    assert lib.fp4_codes_bytes(rows, cols) == 0
    assert lib.fp4_scales_bytes(rows, cols, 32, 1, 0) == 0


@pytest.mark.parametrize("mnk", [(0, 64, 64), (64, 0, 64), (64, 64, 0), (-128, 64, 64)])
def test_empty_gemm_rejected(lib, mnk):
    M, N, K = mnk
    assert lib.fp4_gemm(FAKE, FAKE, None, FAKE, FAKE, None, M, N, K, 0, 32, FAKE, max(N, 1), 0, None) == -1
    assert lib.fp4_gemm_quantize(FAKE, FAKE, None, FAKE, FAKE, None, M, N, K, 0, 32, 0, 32, 0, 0, None, FAKE, FAKE, 0,
                                 None) == -1
