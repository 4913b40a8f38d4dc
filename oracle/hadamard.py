"""Block-diagonal Hadamard rotation (oracle side).

"Bridging the Gap Between Promise and Performance for Microscaling FP4
Quantization", Abstract: block-wise Hadamard transforms, fused into the weights
offline and computed online for the activations; its summary post, item 3:
block-diagonal Hadamard rotations of the activations at inference.

Readings taken (the pages give neither order, normalisation nor signs):
Sylvester order, H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]], so that
H[i, j] = (-1)**popcount(i & j); normalised by 1/sqrt(b); no random sign flips;
blocks are contiguous along the rotated axis starting at index 0; block sizes
b in {16, 32, 64, 128}.  The oracle forms the dense matrix and multiplies in
fp64 (no butterflies), so a reader can check it against the definition.
"""
from __future__ import annotations

import numpy as np


def sylvester(n: int) -> np.ndarray:
    """Unnormalised Sylvester Hadamard matrix of order n (a power of two), by the recursion."""
    if n < 1 or n & (n - 1):
        raise ValueError("order must be a power of two")
    h = np.ones((1, 1), dtype=np.float64)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def block_hadamard(x: np.ndarray, b: int, axis: int = 1) -> np.ndarray:
    """x' = x . (H_b / sqrt(b)) on every contiguous b-block along `axis`, in fp64."""
    x = np.asarray(x, dtype=np.float64)
    if axis == 0:
        return block_hadamard(x.T, b, axis=1).T
    n, L = x.shape
    if L % b:
        raise ValueError("rotated axis length must be a multiple of the Hadamard block")
    h = sylvester(b) / np.sqrt(np.float64(b))
    return (x.reshape(n, L // b, b) @ h).reshape(n, L)
