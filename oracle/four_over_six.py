"""Four-over-six adaptive block scaling for NVFP4 (oracle side).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py): nothing in the product path
imports this.

Source: "Four Over Six: More Accurate NVFP4 Quantization with Adaptive Block
Scaling", Abstract (listed on the "FP4 All the Way" page): for some blocks,
scaling to the smaller FP4 value 4 instead of 6 spreads the representable
values more evenly.

Readings (the page gives no selection rule or arithmetic):
1. Every NVFP4 block has two candidate scale bytes: the standard one,
   sb6 = E4M3_RNE_sat(fp32(fp32(amax_b / 6) / s_t)), and
   sb4 = E4M3_RNE_sat(fp32(fp32(amax_b / 4) / s_t)), with the same tensor
   scale s_t = amax / 2688 as NVFP4.
2. Each candidate is scored by the squared error of its round-to-nearest
   result: e_i = fp64(x_i) - fp64(d_i), with d_i the NVFP4 dequantization
   fp32(fp32(G[c_i] * sb) * s_t), err = sum of fp64(e_i * e_i) added in element
   order in fp64 (the order and the roundings are fixed so that the choice is
   reproducible bit for bit).
3. The block takes sb4 when err4 < err6 strictly, else sb6 (ties and zero
   blocks keep the standard scale); its codes are then produced with the
   requested rounding (RTN, or SR with the element's Philox word) under the
   chosen scale.
The codes and scale bytes are ordinary NVFP4 (dequantize and GEMM unchanged).
"""
from __future__ import annotations

import numpy as np

from .formats import E2M1_GRID, e2m1_rtn, e2m1_sr, e4m3_decode, e4m3_rne_sat
from .philox import philox_words


def nv_block_candidates(amax_b: np.ndarray, s_t: np.float32):
    """(sb6, sb4): the two candidate E4M3 scale bytes per block."""
    s_t = np.float32(s_t)
    t6 = ((amax_b / np.float32(6.0)).astype(np.float32) / s_t).astype(np.float32)
    t4 = ((amax_b / np.float32(4.0)).astype(np.float32) / s_t).astype(np.float32)
    return e4m3_rne_sat(t6), e4m3_rne_sat(t4)


def _rtn_sq_error(xb: np.ndarray, sb: np.ndarray, s_t: np.float32) -> np.ndarray:
    """Sum over each block of fp64 (x - deq(RTN codes))^2, in element order.  xb [..., bs] fp32."""
    S = (e4m3_decode(sb).astype(np.float32) * s_t).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = (xb / S[..., None]).astype(np.float32)
    c = e2m1_rtn(v)
    mag = E2M1_GRID[c & 7]
    g = np.where(c & 8, -mag, mag)
    d = ((g * e4m3_decode(sb)[..., None]).astype(np.float32) * s_t).astype(np.float32)
    d = np.where((sb == 0)[..., None], np.float32(0), d)
    e = xb.astype(np.float64) - d.astype(np.float64)
    return np.cumsum(e * e, axis=-1)[..., -1]          # sequential fp64 sum in element order


def choose_scales(xb: np.ndarray, s_t: np.float32) -> np.ndarray:
    """Chosen scale byte per block of xb [..., 16] (fp32)."""
    amax_b = np.max(np.abs(xb), axis=-1).astype(np.float32)
    sb6, sb4 = nv_block_candidates(amax_b, s_t)
    err6 = _rtn_sq_error(xb, sb6, s_t)
    err4 = _rtn_sq_error(xb, sb4, s_t)
    pick4 = (err4 < err6) & (amax_b > 0) & (sb4 != 0)
    return np.where(pick4, sb4, sb6).astype(np.uint8)


def quantize_rows_46(xw: np.ndarray, idxw: np.ndarray, rnd: str, seed: int, s_t: np.float32):
    """NVFP4 with four-over-six scales on every row of xw [n, L] (L % 16 == 0): (codes [n, L], bytes)."""
    n, L = xw.shape
    xb = xw.reshape(n, L // 16, 16)
    sb = choose_scales(xb, s_t)
    S = (e4m3_decode(sb).astype(np.float32) * np.float32(s_t)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = (xb / S[..., None]).astype(np.float32)
    if rnd == "rtn":
        codes = e2m1_rtn(v)
    else:
        codes = e2m1_sr(v, philox_words(seed, idxw.reshape(n, L // 16, 16)))
    amax_b = np.max(np.abs(xb), axis=-1)
    codes = np.where(((sb == 0) | (amax_b == 0))[..., None], np.uint8(0), codes)
    return codes.reshape(n, L), sb
