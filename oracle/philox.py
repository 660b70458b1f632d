"""Philox4x32-10 counter-based generator (oracle side; TEST INFRASTRUCTURE ONLY).

Written from the published definition of the Philox family (Salmon, Moraes,
Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11, section 4):
a 4-word counter and a 2-word key; each round multiplies words 0 and 2 by the
constants 0xD2511F53 and 0xCD9E8D57, splits each 64-bit product into hi/lo
halves and recombines them with the other two words and the round key; the key
is bumped by the Weyl constants (0x9E3779B9, 0xBB67AE85) between rounds; ten
rounds.

The sampler of "DiffusionGemma Technical Report" (codemajin.net section 3.3;
aibars.net "Uniform State Diffusion") replaces low-confidence tokens with
uniformly random vocabulary tokens; those draws come from this generator.
"""
from __future__ import annotations

import numpy as np

M0 = np.uint64(0xD2511F53)
M1 = np.uint64(0xCD9E8D57)
W0 = 0x9E3779B9
W1 = 0xBB67AE85
_MASK = np.uint64(0xFFFFFFFF)
_S32 = np.uint64(32)


def philox4x32_10(c0, c1, c2, c3, k0: int, k1: int):
    """Vectorised Philox4x32-10.  Counters are array-likes of uint32 values."""
    c0 = np.asarray(c0, dtype=np.uint64) & _MASK
    c1 = np.asarray(c1, dtype=np.uint64) & _MASK
    c2 = np.asarray(c2, dtype=np.uint64) & _MASK
    c3 = np.asarray(c3, dtype=np.uint64) & _MASK
    ka, kb = k0 & 0xFFFFFFFF, k1 & 0xFFFFFFFF
    for r in range(10):
        if r > 0:
            ka = (ka + W0) & 0xFFFFFFFF
            kb = (kb + W1) & 0xFFFFFFFF
        p0 = c0 * M0          # < 2^64, exact in uint64
        p1 = c2 * M1
        hi0, lo0 = p0 >> _S32, p0 & _MASK
        hi1, lo1 = p1 >> _S32, p1 & _MASK
        c0, c1, c2, c3 = (hi1 ^ c1 ^ np.uint64(ka), lo1, hi0 ^ c3 ^ np.uint64(kb), lo0)
    return c0, c1, c2, c3


def uniform_token(word0, vocab: int):
    """Map a 32-bit draw to a token uniform over [0, vocab)."""
    w = np.asarray(word0, dtype=np.uint64)
    if vocab & (vocab - 1) == 0:
        return (w & np.uint64(vocab - 1)).astype(np.int64)
    return ((w * np.uint64(vocab)) >> _S32).astype(np.int64)
