"""Philox4x32-10 counter-based generator (oracle side).

The pages ask for stochastic rounding in the backward/update passes ("FP4 All
the Way", Abstract) but give no generator.  Reading taken: the counter-based
Philox4x32 with 10 rounds, as published by Salmon, Moraes, Dror and Shaw,
"Parallel random numbers: as easy as 1, 2, 3" (SC'11), keyed by the seed and
counted by the element index:

* key     = (seed mod 2**32, seed >> 32)
* counter = (j mod 2**32, j >> 32, 0, 0) with j = idx >> 2
* the element with linear index idx (row-major position in the input tensor
  as stored, whatever the quantization axis) takes output word (idx & 3).

Round function (S-box on two 32x32->64 multiplies), with the published
multipliers and Weyl key increments:
  (hi0, lo0) = M0 * c0,  (hi1, lo1) = M1 * c2
  c <- (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0);   then k <- k + (W0, W1)
"""
from __future__ import annotations

import numpy as np

M0 = 0xD2511F53
M1 = 0xCD9E8D57
W0 = 0x9E3779B9
W1 = 0xBB67AE85
MASK = 0xFFFFFFFF


def philox4x32_10(counter, key, rounds: int = 10) -> np.ndarray:
    """counter: (4, n) uint32-valued array; key: (k0, k1).  Returns (4, n) uint32."""
    c = [np.asarray(counter[i], dtype=np.uint64) & MASK for i in range(4)]
    k0 = np.uint64(int(key[0]) & MASK)
    k1 = np.uint64(int(key[1]) & MASK)
    m0, m1 = np.uint64(M0), np.uint64(M1)
    for rnd in range(rounds):
        p0 = m0 * c[0]                       # < 2**64, exact in uint64
        p1 = m1 * c[2]
        hi0, lo0 = p0 >> np.uint64(32), p0 & np.uint64(MASK)
        hi1, lo1 = p1 >> np.uint64(32), p1 & np.uint64(MASK)
        c = [hi1 ^ c[1] ^ k0, lo1, hi0 ^ c[3] ^ k1, lo0]
        if rnd != rounds - 1:
            k0 = np.uint64((int(k0) + W0) & MASK)
            k1 = np.uint64((int(k1) + W1) & MASK)
    return np.stack([x.astype(np.uint32) for x in c])


def philox_words(seed: int, idx) -> np.ndarray:
    """32-bit random word of each linear element index under `seed`."""
    idx = np.asarray(idx, dtype=np.uint64)
    flat = idx.reshape(-1)
    j = flat >> np.uint64(2)
    uniq, inv = np.unique(j, return_inverse=True)
    ctr = np.stack([uniq & np.uint64(MASK), uniq >> np.uint64(32),
                    np.zeros_like(uniq), np.zeros_like(uniq)])
    out = philox4x32_10(ctr, (seed & MASK, (seed >> 32) & MASK))
    words = out[(flat & np.uint64(3)).astype(np.int64), inv]
    return words.reshape(idx.shape)
