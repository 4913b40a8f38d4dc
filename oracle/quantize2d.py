"""Two-dimensional (square-tile) block quantization of a matrix (oracle side).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py): nothing in the product path
imports this.

Source: "Pretraining Large Language Models with NVFP4", Abstract (listed on the
"FP4 All the Way" page): a two-dimensional quantization scheme gives the
weights one consistent representation in the forward and the backward pass.

Readings (the page gives no tile shape or arithmetic):
1. The tile is square, block x block elements -- 16 x 16 for NVFP4, 32 x 32 for
   MXFP4 -- so that each tile row is one 1-D block of W and each tile column one
   1-D block of W^T.
2. The tile's scale comes from the tile's amax exactly as a 1-D block's scale
   comes from the block's amax (`quantize` readings 2 and 3, the same tensor
   scale for NVFP4).
3. Every element is scaled and rounded once (RTN, or SR with the Philox word of
   its row-major index in the input), so W's codes (packed along its rows) and
   W^T's codes (packed along W's columns) are the same codes, transposed, and
   every row or column segment of a tile carries the tile's scale byte.
"""
from __future__ import annotations

import numpy as np

from .formats import e2m1_rtn, e2m1_sr, e4m3_decode, e4m3_rne_sat, mx_scale_exponent
from .philox import philox_words
from .quantize import FMT_BLOCK, _bf16_to_f32, nv_tensor_scale, pack_nibbles


def quantize_2d(x_bits, fmt: str = "nvfp4", rnd: str = "rtn", seed: int = 0, tensor_scale=None):
    """bf16 bit patterns x[R, C] (R, C multiples of the block) -> dict with
    codes [R, C/2], scales [R, C/bs] (W along its rows), codes_t [C, R/2],
    scales_t [C, R/bs] (W^T along its rows), tensor_scale (NV) or None."""
    bs = FMT_BLOCK[fmt]
    x = _bf16_to_f32(x_bits)
    R, C = x.shape
    if R % bs or C % bs:
        raise ValueError("both dimensions must be multiples of the block size")
    tr, tc = R // bs, C // bs
    tiles = x.reshape(tr, bs, tc, bs)
    amax_t = np.max(np.abs(tiles), axis=(1, 3)).astype(np.float32)          # [tr, tc]
    s_t = None
    if fmt == "mxfp4":
        E = mx_scale_exponent(amax_t)
        tile_bytes = (E + 127).astype(np.uint8)
        S = np.ldexp(np.float64(1.0), E)                                      # exact powers of two
        v = (tiles.astype(np.float64) / S[:, None, :, None]).astype(np.float32)
        zero = amax_t == 0
    else:
        s_t = np.float32(tensor_scale) if tensor_scale is not None else nv_tensor_scale(x)
        t = ((amax_t / np.float32(6.0)).astype(np.float32) / s_t).astype(np.float32)
        tile_bytes = e4m3_rne_sat(t)
        S = (e4m3_decode(tile_bytes).astype(np.float32) * s_t).astype(np.float32)
        with np.errstate(divide="ignore", invalid="ignore"):
            v = (tiles / S[:, None, :, None]).astype(np.float32)
        zero = (tile_bytes == 0) | (amax_t == 0)
    v = v.reshape(R, C)
    if rnd == "rtn":
        codes = e2m1_rtn(v)
    else:
        idx = np.arange(R, dtype=np.int64)[:, None] * C + np.arange(C, dtype=np.int64)[None, :]
        codes = e2m1_sr(v, philox_words(seed, idx))
    zero_el = np.repeat(np.repeat(zero, bs, axis=0), bs, axis=1)
    codes = np.where(zero_el, np.uint8(0), codes).astype(np.uint8)
    return {
        "codes": pack_nibbles(codes),
        "scales": np.repeat(tile_bytes, bs, axis=0),                          # [R, C/bs]
        "codes_t": pack_nibbles(np.ascontiguousarray(codes.T)),
        "scales_t": np.repeat(np.ascontiguousarray(tile_bytes.T), bs, axis=0),  # [C, R/bs]
        "tensor_scale": s_t,
    }
