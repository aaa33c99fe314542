"""Philox4x32-10, the counter-based generator of Salmon, Moraes, Dror and Shaw,
"Parallel Random Numbers: As Easy as 1, 2, 3" (SC 2011), written from its
published definition for the oracle's dropout masks.

TEST INFRASTRUCTURE ONLY (same rule as the rest of ``oracle/``): the CUDA
path implements the same published generator in its own code; the two share
nothing.

One call maps a 128-bit counter (c0, c1, c2, c3) and a 64-bit key (k0, k1)
to four 32-bit words by ten rounds of

    (hi0, lo0) = M0 * c0,  (hi1, lo1) = M1 * c2      (64-bit products)
    (c0, c1, c2, c3) <- (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0)

with the key advanced by the Weyl constants (W0, W1) after every round but
the last. The constants are the paper's.
"""

from __future__ import annotations

import numpy as np

M0 = np.uint64(0xD2511F53)
M1 = np.uint64(0xCD9E8D57)
W0 = np.uint64(0x9E3779B9)
W1 = np.uint64(0xBB67AE85)
MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Element-wise Philox4x32-10 over arrays of uint32-valued counters and
    keys (any broadcastable shapes). Returns four uint32 arrays."""
    c0, c1, c2, c3, k0, k1 = (np.asarray(x, dtype=np.uint64) & MASK32 for x in (c0, c1, c2, c3, k0, k1))
    for r in range(10):
        p0 = M0 * c0
        p1 = M1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & MASK32
        c0, c1, c2, c3 = (hi1 ^ c1 ^ k0) & MASK32, lo1, (hi0 ^ c3 ^ k1) & MASK32, lo0
        if r < 9:
            k0 = (k0 + W0) & MASK32
            k1 = (k1 + W1) & MASK32
    return tuple(x.astype(np.uint32) for x in (c0, c1, c2, c3))
