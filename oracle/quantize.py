"""MXFP4 / NVFP4 block quantization and dequantization (oracle side).

What the method computes (sources by page and section):
* "FP4 All the Way: Fully Quantized Training of LLMs", Abstract: each block of
  16 E2M1 values shares an E4M3 scale (NVFP4); weights, activations and
  gradients are all quantized; round-to-nearest forward, stochastic rounding
  backward/update.
* "Bridging the Gap Between Promise and Performance for Microscaling FP4
  Quantization", Abstract: MXFP4 with power-of-two scales (32-element groups
  in the MX convention); NVFP4's small groups.
* "Oscillation-Reduced MXFP4 Training for Vision Transformers", Abstract: MX
  is fine-grained per-group scaling.

Readings taken where the pages are silent (plainest reading, OCP MX v1.0):
1. Input bf16 widened to fp32 (exact).
2. MXFP4 (block 32): amax_b = max |x|; E = clamp(floor(log2 amax_b) - 2,
   -127, 127) (E = -127 for amax_b = 0); scale 2**E; byte E + 127.
3. NVFP4 (block 16): s_t = fp32(amax_tensor / 2688) (2688 = 6 * 448), 1.0 when
   amax_tensor = 0, unless the caller gives s_t; per block
   t = fp32(fp32(amax_b / 6) / s_t); sb = E4M3_RNE(min(t, 448));
   S_b = fp32(sb * s_t).
4. v = fp32(x / S_b) (correctly rounded division; exact for MX).
5. RTN: nearest E2M1, ties to even code, saturate at 6, sign kept.
   SR: see `formats.e2m1_sr`, random word from `philox.philox_words` at the
   element's row-major index in the input as stored.
6. Blocks whose scale is zero (amax_b = 0, or NV sb = 0) get all codes +0.
7. Packing: byte j of a row holds element 2j in the low nibble and 2j+1 in the
   high nibble.  axis=1 quantizes along columns (output [rows, cols/2]);
   axis=0 quantizes along rows and writes the transpose (output
   [cols, rows/2]), so the contraction axis is always the packed one.
8. Optional block-Hadamard rotation (see `hadamard`) is applied along the
   quantization axis before step 2, in fp64, and rounded to fp32.
"""
from __future__ import annotations

import numpy as np

from .formats import (E2M1_GRID, e2m1_rtn, e2m1_sr, e4m3_decode, e4m3_rne_sat,
                      mx_scale_exponent)
from .philox import philox_words
from .hadamard import block_hadamard

FMT_BLOCK = {"mxfp4": 32, "nvfp4": 16}


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[..., 0::2] & 0xF) | ((codes[..., 1::2] & 0xF) << 4)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = packed & 0xF
    out[..., 1::2] = packed >> 4
    return out


def _bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def nv_tensor_scale(x32: np.ndarray) -> np.float32:
    """s_t = amax / (6 * 448) in fp32; 1.0 for an all-zero tensor."""
    amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(amax / np.float32(2688.0))


def _quantize_rows(xw: np.ndarray, idxw: np.ndarray, fmt: str, bs: int, rnd: str, seed: int,
                   s_t: np.float32, mx_clip=None):
    """Quantize every row of xw (fp32 [n, L], L % bs == 0) in contiguous bs-blocks.  mx_clip: the
    MXFP4 exponent's clip threshold (`mse_grid` reading 6), None for the OCP rule."""
    n, L = xw.shape
    xb = xw.reshape(n, L // bs, bs)
    amax_b = np.max(np.abs(xb), axis=2).astype(np.float32)                 # [n, G]
    if fmt == "mxfp4":
        if mx_clip is None:
            E = mx_scale_exponent(amax_b)
        else:
            from .mse_grid import mx_scale_exponent_clip
            E = mx_scale_exponent_clip(amax_b, mx_clip)
        scale_bytes = (E + 127).astype(np.uint8)
        S = np.ldexp(np.float64(1.0), E)                                      # exact powers of two
        v = (xb.astype(np.float64) / S[..., None]).astype(np.float32)        # exact quotient, rounded to fp32
        zero_block = amax_b == 0
    else:
        t = ((amax_b / np.float32(6.0)).astype(np.float32) / s_t).astype(np.float32)
        sb = e4m3_rne_sat(t)
        scale_bytes = sb
        S_b = (e4m3_decode(sb).astype(np.float32) * s_t).astype(np.float32)
        with np.errstate(divide="ignore", invalid="ignore"):
            v = (xb / S_b[..., None]).astype(np.float32)
        zero_block = (sb == 0) | (amax_b == 0)
    if rnd == "rtn":
        codes = e2m1_rtn(v)
    else:
        r = philox_words(seed, idxw.reshape(n, L // bs, bs))
        codes = e2m1_sr(v, r)
    codes = np.where(zero_block[..., None], np.uint8(0), codes)
    return codes.reshape(n, L), scale_bytes


def quantize_values(x32, fmt: str = "mxfp4", block: int | None = None, axis: int = 1, rnd: str = "rtn",
                    seed: int = 0, tensor_scale=None, idx_base: int = 0, idx_cols: int | None = None):
    """Steps 2-7 on fp32 values x32 [rows, cols] (already widened/rotated).

    The Philox index of element (r, c) is idx_base + r * idx_cols + c (idx_cols
    defaults to cols), so a row slice of a larger tensor can be quantized with
    its global indices.  For NVFP4 without `tensor_scale`, s_t comes from x32.
    fmt "nvfp4_4o6" is NVFP4 with four-over-six block scales (`four_over_six`); fmt "mxfp4_gs" is
    MXFP4 whose block exponents use the MSE-fitted clip threshold (`mse_grid`, readings 6-7).
    """
    four_six = fmt == "nvfp4_4o6"
    mx_clip = None
    if fmt == "mxfp4_gs":
        from .mse_grid import MX_GRID_CLIP
        mx_clip = MX_GRID_CLIP
        fmt = "mxfp4"
    fmt = "nvfp4" if four_six else fmt
    bs = block or FMT_BLOCK[fmt]
    if (fmt, bs) not in (("mxfp4", 32), ("nvfp4", 16)):
        raise ValueError("supported: (mxfp4, 32), (nvfp4, 16)")
    x = np.asarray(x32, dtype=np.float32)
    R, C = x.shape
    ic = C if idx_cols is None else idx_cols
    idx = (np.int64(idx_base) + np.arange(R, dtype=np.int64)[:, None] * ic
           + np.arange(C, dtype=np.int64)[None, :])
    xw, idxw = (x, idx) if axis == 1 else (x.T, idx.T)
    if xw.shape[1] % bs:
        raise ValueError("quantization axis length must be a multiple of the block size")
    s_t = None
    if fmt == "nvfp4":
        s_t = np.float32(tensor_scale) if tensor_scale is not None else nv_tensor_scale(x)
    if four_six:
        from .four_over_six import quantize_rows_46
        codes, scales = quantize_rows_46(np.ascontiguousarray(xw), np.ascontiguousarray(idxw), rnd, seed, s_t)
    else:
        codes, scales = _quantize_rows(np.ascontiguousarray(xw), np.ascontiguousarray(idxw),
                                       fmt, bs, rnd, seed, s_t, mx_clip)
    return {"codes": pack_nibbles(codes), "scales": scales, "tensor_scale": s_t}


def quantize(x_bits, fmt: str = "mxfp4", block: int | None = None, axis: int = 1,
             rnd: str = "rtn", seed: int = 0, tensor_scale=None, had_block: int | None = None,
             idx_base: int = 0, idx_cols: int | None = None):
    """Quantize a bf16 tensor (given as uint16 bit patterns, [rows, cols]).

    Returns a dict with
      codes        uint8 [out_rows, L/2] packed E2M1 codes (out_rows = rows, L = cols
                   for axis 1; out_rows = cols, L = rows for axis 0),
      scales       uint8 [out_rows, L/block] E8M0 (MX) or E4M3 (NV) bytes, row-major,
      tensor_scale np.float32 s_t (NV) or None (MX),
      rotated      fp32 [rows, cols] rotated input (only when had_block is given).
    """
    x = _bf16_to_f32(x_bits)
    rotated = None
    if had_block:
        x = block_hadamard(x.astype(np.float64), had_block, axis=axis).astype(np.float32)
        rotated = x
    out = quantize_values(x, fmt, block, axis, rnd, seed, tensor_scale, idx_base, idx_cols)
    out["rotated"] = rotated
    return out


def dequantize(codes_packed, scales, fmt: str = "mxfp4", block: int | None = None,
               tensor_scale=None, out: str = "f32") -> np.ndarray:
    """Packed codes [n, L/2] + row-major scales [n, L/block] -> fp32 [n, L].

    MX: G[c] * 2**E, exact.  NV: fp32(fp32(G[c] * sb) * s_t), where G[c] * sb is
    exact.  out="bf16" additionally rounds to bf16 (RNE) and returns the bits.
    """
    bs = block or FMT_BLOCK[fmt]
    c = unpack_nibbles(codes_packed)
    n, L = c.shape
    mag = E2M1_GRID[c & 7]
    val = np.where(c & 8, -mag, mag).reshape(n, L // bs, bs)
    scales = np.asarray(scales, dtype=np.uint8)
    if fmt == "mxfp4":
        E = scales.astype(np.int64) - 127
        y = (val * np.ldexp(np.float64(1.0), E)[..., None]).astype(np.float32)
    else:
        sb = e4m3_decode(scales)
        y = ((val * sb[..., None]).astype(np.float32) * np.float32(tensor_scale)).astype(np.float32)
    y = y.reshape(n, L)
    if out == "bf16":
        import ml_dtypes
        return y.astype(ml_dtypes.bfloat16).view(np.uint16)
    return y
