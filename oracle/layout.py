"""Tensor-core scale-factor layout (oracle side).

The pages print no layout.  Besides the plain row-major `[rows, K/block]`
layout, the quantizer can write its scale bytes straight into the layout that
Blackwell's block-scaled MMA consumes (PTX ISA, tcgen05 block scaling: scale
factors move to tensor memory in 32-lane x 16-byte chunks that are replicated
over the four lane quadrants).  Written out from that public description:

* rows are padded to a multiple of 128 and scale columns (k-groups) to a
  multiple of 4; padding bytes are 0;
* the padded matrix is cut into 128x4 tiles, stored tile-row-major with the
  k-tile index fastest: tile (rb, kb) starts at byte ((rb * G4) + kb) * 512,
  G4 = padded k-groups / 4;
* inside a tile, row r (0..127) and k-group g (0..3) sit at byte
  (r % 32) * 16 + (r // 32) * 4 + g.
"""
from __future__ import annotations

import numpy as np


def _round_up(a: int, b: int) -> int:
    return (a + b - 1) // b * b


def sf_mma_bytes(rows: int, groups: int) -> int:
    return _round_up(rows, 128) * _round_up(groups, 4)


def _offsets(rows: int, groups: int) -> np.ndarray:
    g4 = _round_up(groups, 4) // 4
    r = np.arange(rows)[:, None]
    g = np.arange(groups)[None, :]
    return ((r // 128) * g4 + g // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (g % 4)


def sf_to_mma(scales: np.ndarray) -> np.ndarray:
    """Row-major scale bytes [rows, groups] -> flat uint8 array in the MMA layout."""
    scales = np.asarray(scales, dtype=np.uint8)
    rows, groups = scales.shape
    out = np.zeros(sf_mma_bytes(rows, groups), dtype=np.uint8)
    out[_offsets(rows, groups)] = scales
    return out


def sf_from_mma(flat: np.ndarray, rows: int, groups: int) -> np.ndarray:
    flat = np.asarray(flat, dtype=np.uint8).reshape(-1)
    return flat[_offsets(rows, groups)]
