"""Element and scale formats of microscaling FP4 (oracle side).

The pages name the formats but print no encodings:
* "FP4 All the Way: Fully Quantized Training of LLMs", Abstract: FP4 values are
  E2M1; NVFP4 blocks of 16 share an E4M3 scale.
* "Bridging the Gap Between Promise and Performance for Microscaling FP4
  Quantization", Abstract: MXFP4 uses power-of-two scales.

Readings taken (OCP Microscaling v1.0 conventions, the plainest reading):
* E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0, no Inf/NaN.
  Magnitudes by code 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6.
* E8M0 (MX scale byte b): 2**(b - 127); b = 0xFF is NaN.
* E4M3 (NV scale byte, "E4M3FN"): bias 7, subnormals kept, max 448, 0x7F NaN.
* Round-to-nearest: nearest representable value, ties to the even code
  (mantissa LSB 0); magnitudes beyond the largest value saturate; the sign of
  the input is kept (so -tiny -> code 0x8, i.e. -0).
"""
from __future__ import annotations

import numpy as np


def _e2m1_value(code: int) -> float:
    """Value of a 4-bit E2M1 code, straight from the bit fields."""
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = 0.5 * m if e == 0 else 2.0 ** (e - 1) * (1.0 + 0.5 * m)
    return -mag if s else mag


#: E2M1 magnitudes, index = 3-bit magnitude code.
E2M1_GRID = np.array([_e2m1_value(c) for c in range(8)], dtype=np.float64)


def e2m1_decode(codes) -> np.ndarray:
    """4-bit codes (0..15) -> float64 values (-0.0 for code 8)."""
    codes = np.asarray(codes, dtype=np.uint8) & 0xF
    mag = E2M1_GRID[codes & 7]
    return np.where(codes & 8, -mag, mag)


def _nearest_even(mag: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Index of the nearest entry of the ascending `table` to each `mag`,
    ties going to the even index; values beyond the ends clamp to the ends.
    Distances are formed in fp64, where they are exact for fp32 inputs near
    the table entries, so ties are detected exactly."""
    mag = np.asarray(mag, dtype=np.float64)
    hi = np.searchsorted(table, mag, side="left")            # table[hi-1] < mag <= table[hi]
    hi = np.clip(hi, 1, len(table) - 1)
    lo = hi - 1
    d_lo = mag - table[lo]
    d_hi = table[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(mag >= table[-1], len(table) - 1, idx)
    idx = np.where(mag <= table[0], 0, idx)
    return idx


def e2m1_rtn(v) -> np.ndarray:
    """Round fp32 values to E2M1 codes: nearest, ties to even code, saturating at 6."""
    v = np.asarray(v, dtype=np.float32)
    mag_code = _nearest_even(np.abs(v.astype(np.float64)), E2M1_GRID).astype(np.uint8)
    return mag_code | (np.signbit(v).astype(np.uint8) << 3)


def e2m1_sr(v, r) -> np.ndarray:
    """Stochastic rounding of fp32 values to E2M1 codes with 32-bit random words r.

    Reading (the pages only say "stochastic rounding for backward and update
    passes", "FP4 All the Way", Abstract): with lo <= |v| < hi adjacent grid
    points, p = (|v| - lo) / (hi - lo) computed in fp32 (exact here), round up
    to hi iff r < ceil(p * 2**32); |v| >= 6 gives 6; the sign is kept.
    """
    v = np.asarray(v, dtype=np.float32)
    r = np.asarray(r, dtype=np.uint64)
    a = np.abs(v)
    # lo index: largest grid point <= |v|
    lo_i = np.searchsorted(E2M1_GRID, a.astype(np.float64), side="right") - 1
    lo_i = np.clip(lo_i, 0, 7)
    sat = a >= np.float32(6.0)
    hi_i = np.minimum(lo_i + 1, 7)
    lo = E2M1_GRID[lo_i].astype(np.float32)
    hi = E2M1_GRID[hi_i].astype(np.float32)
    width = np.where(sat, np.float32(1.0), hi - lo).astype(np.float32)
    with np.errstate(invalid="ignore"):
        p = ((a - lo) / width).astype(np.float32)                   # fp32, exact
        p = np.where(np.isfinite(p), p, np.float32(0))              # non-finite v: saturated above
    thr = np.ceil(p.astype(np.float64) * 2.0 ** 32).astype(np.uint64)  # p*2^32 exact in fp64
    up = (r < thr) & ~sat
    mag_code = np.where(sat, 7, np.where(up, hi_i, lo_i)).astype(np.uint8)
    return mag_code | (np.signbit(v).astype(np.uint8) << 3)


# --- E4M3 (NVFP4 block scale) -------------------------------------------------

def _e4m3_value(byte: int) -> float:
    s, e, m = (byte >> 7) & 1, (byte >> 3) & 0xF, byte & 7
    if e == 0xF and m == 7:
        return float("nan")
    mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


_E4M3_POS = np.array([_e4m3_value(b) for b in range(0x7F)], dtype=np.float64)  # 0x00..0x7E, ascending
E4M3_MAX = _E4M3_POS[-1]   # 448


def e4m3_decode(b) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint8)
    table = np.array([_e4m3_value(i) for i in range(256)], dtype=np.float64)
    return table[b]


def e4m3_rne_sat(t) -> np.ndarray:
    """Non-negative fp32 -> E4M3 byte: values above 448 clamp to 448 first, then
    nearest representable with ties to even mantissa (subnormals kept)."""
    t = np.asarray(t, dtype=np.float32).astype(np.float64)
    t = np.minimum(t, E4M3_MAX)
    return _nearest_even(t, _E4M3_POS).astype(np.uint8)


# --- E8M0 (MXFP4 block scale) ---------------------------------------------------

def mx_scale_exponent(amax) -> np.ndarray:
    """Shared power-of-two exponent E of an MXFP4 block, as an int64.

    Reading (OCP MX v1.0, the pages give only "power-of-two scale"):
    E = floor(log2(amax)) - emax_elem with emax_elem = 2 for E2M1 (6 = 1.5 * 2**2),
    clamped to the E8M0 range [-127, 127]; amax = 0 gives E = -127 (byte 0x00).
    floor(log2) is taken exactly from frexp (mantissa in [0.5, 1)).
    """
    amax = np.asarray(amax, dtype=np.float32)
    _, ex = np.frexp(amax.astype(np.float64))
    e = ex.astype(np.int64) - 1
    E = np.clip(e - 2, -127, 127)
    return np.where(amax == 0, -127, E)
