"""Reference for the block-scaled FP4 x FP4 GEMM (oracle side).

"Bridging the Gap Between Promise and Performance for Microscaling FP4
Quantization", Abstract: FP4 GEMM kernels on B200 consuming MXFP4/NVFP4
operands; "Oscillation-Reduced MXFP4 Training for Vision Transformers",
Abstract: MX matmuls on Blackwell.

Both operands are K-major ("TN"): A codes [M, K/2] with scales [M, K/block],
B codes [N, K/2] with scales [N, K/block]; Y[M, N] = alpha * sum_k a[m,k] b[n,k]
where a = G[code] * block_scale (MX: 2**E, NV: the E4M3 value) and alpha = 1
(MX) or s_tA * s_tB (NV).  Reading: accumulation is exact here (fp64; for the
small pinned cases it is exact, see the tests), and the acceptance bound per
element is |dY| <= 1e-5 * sum_k |alpha * a b|, which `gemm_ref` returns too.
"""
from __future__ import annotations

import numpy as np

from .formats import E2M1_GRID, e4m3_decode
from .quantize import unpack_nibbles, FMT_BLOCK


def deq_for_gemm(codes_packed, scales, fmt: str, block: int | None = None, rows=None) -> np.ndarray:
    """Operand values the tensor core multiplies (block scale applied, no tensor scale), fp64."""
    bs = block or FMT_BLOCK[fmt]
    c = unpack_nibbles(codes_packed if rows is None else np.asarray(codes_packed)[rows])
    s = np.asarray(scales, dtype=np.uint8)
    if rows is not None:
        s = s[rows]
    n, K = c.shape
    mag = E2M1_GRID[c & 7]
    val = np.where(c & 8, -mag, mag).reshape(n, K // bs, bs)
    if fmt == "mxfp4":
        sc = np.ldexp(np.float64(1.0), s.astype(np.int64) - 127)
    else:
        sc = e4m3_decode(s)
    return (val * sc[..., None]).reshape(n, K)


def _alpha(fmt: str, a_ts, b_ts) -> float:
    return 1.0 if fmt == "mxfp4" else float(np.float64(a_ts) * np.float64(b_ts))


def gemm_ref(qa: dict, qb: dict, fmt: str, block: int | None = None):
    """Full fp64 reference.  qa/qb are `quantize` outputs (or dicts with codes/scales/tensor_scale).
    Returns (Y [M,N] fp64, bound [M,N] fp64)."""
    a = deq_for_gemm(qa["codes"], qa["scales"], fmt, block)
    b = deq_for_gemm(qb["codes"], qb["scales"], fmt, block)
    al = _alpha(fmt, qa.get("tensor_scale"), qb.get("tensor_scale"))
    return al * (a @ b.T), abs(al) * (np.abs(a) @ np.abs(b).T)


def gemm_ref_rows(qa: dict, qb: dict, fmt: str, rows, block: int | None = None):
    """Reference for selected output rows (all columns)."""
    a = deq_for_gemm(qa["codes"], qa["scales"], fmt, block, rows=rows)
    b = deq_for_gemm(qb["codes"], qb["scales"], fmt, block)
    al = _alpha(fmt, qa.get("tensor_scale"), qb.get("tensor_scale"))
    return al * (a @ b.T), abs(al) * (np.abs(a) @ np.abs(b).T)


def gemm_ref_cols(qa: dict, qb: dict, fmt: str, cols, block: int | None = None):
    """Reference for selected output columns (all rows); returns [M, len(cols)]."""
    a = deq_for_gemm(qa["codes"], qa["scales"], fmt, block)
    b = deq_for_gemm(qb["codes"], qb["scales"], fmt, block, rows=cols)
    al = _alpha(fmt, qa.get("tensor_scale"), qb.get("tensor_scale"))
    return al * (a @ b.T), abs(al) * (np.abs(a) @ np.abs(b).T)
