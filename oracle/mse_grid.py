"""MSE-fitted FP4 grid scales (oracle side).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py): nothing in the product path
imports this.

Source: the summary post of "Bridging the Gap Between Promise and Performance
for Microscaling FP4 Quantization" (its MR-GPTQ list, item 1): the quantization
grid is made MSE-effective by optimizing it alternately at the scale of each
block and of the whole tensor, which helps NVFP4 without rotations a great
deal; for MXFP4 with Hadamard rotations one fixed grid scale serves every
model.  The page names the idea only; the readings below make it computable.

Readings, NVFP4 (the alternating search):
1. Objective: the squared error of the round-to-nearest result of a block,
   err_b(sb, s_t) = sum_i (fp64(x_i) - fp64(d_i))^2 with
   d_i = fp32(fp32(G[c_i] * sb) * s_t), c_i the RTN code of fp32(x_i / fp32(sb * s_t)),
   added in fp64 in element order (a zero byte dequantizes to 0) -- the score
   four-over-six uses.
2. Block step (s_t fixed): b6 = the standard NVFP4 byte of the block under s_t
   (quantize reading 3).  b6 = 0 keeps 0.  Otherwise the candidates are the
   bytes b6-8 .. b6+8 clipped to [1, 126] -- the eight E4M3 values below and
   above the standard one, an octave either way for normal bytes -- and the
   block takes the candidate of least error, ties
   going to the one met first in the order b6, b6-1, b6+1, b6-2, b6+2, ...
3. Tensor step: the candidates are s_k = fp32(s_t * (1 + k/64)), k = -8 .. 8,
   each scored after its own block step (with the bytes held fixed instead, the
   current s_t always wins: the bytes were just fitted to it).  The score is the
   integer Q(s_k) = sum over blocks of floor(err_b(beta_b(s_k), s_k) * 2^P), with
   beta_b(s_k) block b's byte from a block step under s_k, P = 80 - 2 e_A and
   e_A = floor(log2 amax) of the tensor: each term is below 2^87 (the RTN point
   is never farther from x than 0 is, so |x - d| <= |x| up to d's own
   rounding, and err_b <= 16 amax^2) and the sum is exact in any order; the
   truncation drops less than amax^2 * 2^-80 per block.  The least Q wins, ties
   going to the smallest |k|, then to k < 0; the bytes are those of the winner.
4. Schedule: s_t = amax / 2688 (quantize reading 3) and a block step, then
   `iters` tensor steps (0 <= iters <= 8), each searching around the last s_t.
5. Output: ordinary NVFP4 -- the final s_t and bytes, codes by RTN or SR (the
   Philox word of the element) under them.  An all-zero tensor gives s_t = 1,
   bytes 0, codes 0.  Blocks run along the rows (axis 1).

Readings, MXFP4 (the fixed grid scale):
6. The grid scale is read as the clip threshold T of the block exponent: E is
   the smallest exponent whose grid still reaches T * 2^E >= amax_b, i.e.
   E = floor(log2 amax_b) - 2 + [amax_b > T * 2^(floor(log2 amax_b) - 2)],
   clamped to [-127, 127] (E = -127 for amax_b = 0).  T = 8 is the OCP rule
   (floor(log2 amax_b) - 2, elements in (6, 8) clip to 6); T = 6 never clips.
7. T = MX_GRID_CLIP = 7.25, the value on a 1/16 grid of [6, 8] that minimises
   the mean squared RTN error of MXFP4 on block-Hadamard-rotated Gaussian data
   (`fit_mx_grid_clip`; rotated heavy-tailed and outlier-channel data give
   7.0 - 7.25, against 6-10 % more error at T = 8).
"""
from __future__ import annotations

import numpy as np

from .formats import E2M1_GRID, e2m1_rtn, e2m1_sr, e4m3_decode, e4m3_rne_sat
from .four_over_six import _rtn_sq_error
from .philox import philox_words
from .quantize import _bf16_to_f32, nv_tensor_scale, pack_nibbles

MX_GRID_CLIP = np.float32(7.25)
BLOCK_WINDOW = 8                      # block step: bytes b6 - 8 .. b6 + 8
TENSOR_STEPS = np.arange(-8, 9)       # tensor step: s_t * (1 + k / 64)
MAX_ITERS = 8


# ----------------------------------------------------------------- MXFP4 ----

def mx_scale_exponent_clip(amax, T) -> np.ndarray:
    """MXFP4 block exponent under clip threshold T (reading 6), int64."""
    amax = np.asarray(amax, dtype=np.float32).astype(np.float64)
    _, ex = np.frexp(amax)
    e0 = ex.astype(np.int64) - 1                       # floor(log2 amax) for amax > 0
    up = amax > np.float64(T) * np.ldexp(1.0, e0 - 2)
    E = np.clip(e0 - 2 + up.astype(np.int64), -127, 127)
    return np.where(amax == 0, -127, E)


def mx_rtn_mse(x32: np.ndarray, T) -> float:
    """Mean squared RTN error of MXFP4 (block 32 along rows) under clip threshold T, fp64."""
    xb = np.asarray(x32, dtype=np.float32).reshape(-1, 32)
    am = np.max(np.abs(xb), axis=1)
    S = np.ldexp(1.0, mx_scale_exponent_clip(am, T))
    v = (xb.astype(np.float64) / S[:, None]).astype(np.float32)
    c = e2m1_rtn(v)
    mag = E2M1_GRID[c & 7]
    d = np.where(c & 8, -mag, mag) * S[:, None]
    return float(np.mean((xb.astype(np.float64) - d) ** 2))


def fit_mx_grid_clip(x32: np.ndarray, grid=None):
    """The clip threshold on `grid` (default 6, 6 + 1/16, ..., 8) of least `mx_rtn_mse` on x32,
    with the errors of every grid point."""
    grid = np.arange(6.0, 8.0 + 1e-9, 1.0 / 16) if grid is None else np.asarray(grid, dtype=np.float64)
    errs = np.array([mx_rtn_mse(x32, T) for T in grid])
    return np.float32(grid[int(np.argmin(errs))]), grid, errs


# ----------------------------------------------------------------- NVFP4 ----

def _standard_bytes(amax_b: np.ndarray, s_t: np.float32) -> np.ndarray:
    t = ((amax_b / np.float32(6.0)).astype(np.float32) / np.float32(s_t)).astype(np.float32)
    return e4m3_rne_sat(t).astype(np.int64)


def _window_order() -> np.ndarray:
    """Offsets in tie-break order: 0, -1, +1, -2, +2, ..., -8, +8."""
    out = [0]
    for j in range(1, BLOCK_WINDOW + 1):
        out += [-j, j]
    return np.array(out, dtype=np.int64)


def block_step(xb: np.ndarray, s_t: np.float32) -> np.ndarray:
    """Reading 2: the byte of every block of xb [n, 16] (fp32) under tensor scale s_t."""
    amax_b = np.max(np.abs(xb), axis=-1).astype(np.float32)
    b6 = _standard_bytes(amax_b, s_t)
    offs = _window_order()
    cand = np.clip(b6[:, None] + offs[None, :], 1, 126)                   # [n, 17]
    errs = np.stack([_rtn_sq_error(xb, cand[:, j].astype(np.uint8), np.float32(s_t))
                     for j in range(len(offs))], axis=1)
    best = cand[np.arange(len(xb)), np.argmin(errs, axis=1)]              # first minimum in tie order
    return np.where(b6 == 0, 0, best).astype(np.uint8)


def _exact_floor_sum(err: np.ndarray, P: int) -> int:
    """sum floor(err * 2^P) over the array, exactly (each term < 2^90)."""
    w = np.ldexp(np.asarray(err, dtype=np.float64), P)
    w = np.floor(w)
    total = 0
    for j in (2, 1, 0):                                                   # 30-bit limbs, summed in int64
        limb = np.floor(np.ldexp(w, -30 * j))
        w = w - np.ldexp(limb, 30 * j)
        total += int(limb.astype(np.int64).sum()) << (30 * j)
    return total


def tensor_objective(xb: np.ndarray, sb: np.ndarray, s: np.float32, P: int) -> int:
    """Q of blocks xb [n, 16] with bytes sb under tensor scale s (reading 3's sum)."""
    return _exact_floor_sum(_rtn_sq_error(xb, sb, np.float32(s)), P)


def tensor_candidates(s_t: np.float32) -> np.ndarray:
    m = (np.float32(1.0) + TENSOR_STEPS.astype(np.float32) / np.float32(64.0)).astype(np.float32)
    return (np.float32(s_t) * m).astype(np.float32)


def tensor_step(xb: np.ndarray, s_t: np.float32, P: int):
    """Reading 3: (new s_t, its bytes, the scores Q of all candidates in k order)."""
    cands = tensor_candidates(s_t)
    Q, bytes_k = [], []
    for s in cands:
        sb = block_step(xb, s)
        bytes_k.append(sb)
        Q.append(tensor_objective(xb, sb, s, P))
    best = min(range(len(cands)), key=lambda i: (Q[i], abs(int(TENSOR_STEPS[i])), int(TENSOR_STEPS[i])))
    return np.float32(cands[best]), bytes_k[best], Q


def objective_exponent(amax: np.float32) -> int:
    """P = 80 - 2 floor(log2 amax)."""
    _, ex = np.frexp(np.float64(amax))
    return 80 - 2 * (int(ex) - 1)


def mse_search(x32: np.ndarray, iters: int = 1):
    """Readings 2-4 on fp32 x32 [rows, cols] (cols % 16 == 0): (s_t, bytes [rows, cols/16])."""
    if not 0 <= iters <= MAX_ITERS:
        raise ValueError("iters must be in [0, 8]")
    x = np.asarray(x32, dtype=np.float32)
    R, C = x.shape
    if C % 16:
        raise ValueError("cols must be a multiple of 16")
    s_t = nv_tensor_scale(x)
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0)
    xb = x.reshape(R * (C // 16), 16)
    if amax == 0:
        return s_t, np.zeros((R, C // 16), dtype=np.uint8)
    P = objective_exponent(amax)
    sb = block_step(xb, s_t)
    for _ in range(iters):
        s_t, sb, _ = tensor_step(xb, s_t, P)
    return s_t, sb.reshape(R, C // 16)


def quantize_mse(x_bits, rnd: str = "rtn", seed: int = 0, iters: int = 1):
    """NVFP4 quantization (axis 1) with MSE-searched scales (reading 5) of a bf16 tensor given as
    uint16 bit patterns: dict(codes [R, C/2], scales [R, C/16], tensor_scale)."""
    x = _bf16_to_f32(x_bits)
    R, C = x.shape
    s_t, sb = mse_search(x, iters)
    xb = x.reshape(R, C // 16, 16)
    S = (e4m3_decode(sb).astype(np.float32) * s_t).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = (xb / S[..., None]).astype(np.float32)
    if rnd == "rtn":
        codes = e2m1_rtn(v)
    else:
        idx = np.arange(R * C, dtype=np.int64).reshape(R, C // 16, 16)
        codes = e2m1_sr(v, philox_words(seed, idx))
    codes = np.where((sb == 0)[..., None], np.uint8(0), codes)
    return {"codes": pack_nibbles(codes.reshape(R, C)), "scales": sb, "tensor_scale": np.float32(s_t)}
