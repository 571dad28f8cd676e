"""Philox4x32-10 counter-based generator (oracle; test infrastructure only).

Implemented from Salmon, Moraes, Dror & Shaw, "Parallel random numbers: as easy
as 1, 2, 3" (SC'11), section 4: a 4-word counter and a 2-word key; each of the
10 rounds multiplies words 0 and 2 by two fixed 32-bit constants, takes the
high and low halves of the 64-bit products, and mixes them with words 1 and 3
and the round key; the key is advanced by two Weyl constants between rounds.

The stochastic-rounding mode draws its random words here on the CPU side; the
CUDA library draws the same words from its own implementation of the same
published definition, so that both sides see identical bits without passing
them through memory.  Vectorised over numpy arrays of counters.
"""

from __future__ import annotations

import numpy as np

_M0 = np.uint64(0xD2511F53)
_M1 = np.uint64(0xCD9E8D57)
_W0 = 0x9E3779B9
_W1 = 0xBB67AE85
_MASK = np.uint64(0xFFFFFFFF)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Return the four 32-bit output words (uint32 arrays) for counters (c0..c3) and key (k0, k1)."""
    c = [np.asarray(v, np.uint64) & _MASK for v in (c0, c1, c2, c3)]
    c = np.broadcast_arrays(*c)
    c = [a.copy() for a in c]
    key0 = int(k0) & 0xFFFFFFFF
    key1 = int(k1) & 0xFFFFFFFF
    for rnd in range(10):
        if rnd:
            key0 = (key0 + _W0) & 0xFFFFFFFF
            key1 = (key1 + _W1) & 0xFFFFFFFF
        p0 = _M0 * c[0]          # < 2^64, exact in uint64
        p1 = _M1 * c[2]
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK
        c = [hi1 ^ c[1] ^ np.uint64(key0), lo1, hi0 ^ c[3] ^ np.uint64(key1), lo0]
    return [a.astype(np.uint32) for a in c]


def sr_words(seed: int, unit, epoch, n_elems: int) -> np.ndarray:
    """Random words for stochastic rounding of one state tile.

    Element e of tile ``unit`` (= sequence * nheads + head) written by the fold
    that produces ``epoch`` takes word e % 4 of Philox4x32-10 with counter
    (unit, epoch, e // 4, 0) and key (low 32 bits of seed, high 32 bits).
    ``unit`` and ``epoch`` may be arrays (broadcast over leading dims); returns
    uint32 [..., n_elems].
    """
    unit = np.asarray(unit, np.uint64)[..., None]
    epoch = np.asarray(epoch, np.uint64)[..., None]
    blk = np.arange((n_elems + 3) // 4, dtype=np.uint64)
    w = philox4x32_10(unit, epoch, blk, 0, seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    out = np.stack(w, axis=-1)                                    # [..., blocks, 4]
    return out.reshape(out.shape[:-2] + (-1,))[..., :n_elems]
