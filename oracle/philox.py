"""Philox4x32-10 counter-based generator, written from its published definition.

Source: J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw, "Parallel random
numbers: as easy as 1, 2, 3", SC'11 (the Philox-4xW-R family).  One round maps
the counter (x0, x1, x2, x3) under key (k0, k1) to

    (hi(M1*x2) ^ x1 ^ k0,  lo(M1*x2),  hi(M0*x0) ^ x3 ^ k1,  lo(M0*x0))

where hi/lo are the upper/lower W bits of the 2W-bit product; the key is
bumped by the Weyl constants (W0, W1) after every round.  Ten rounds.

TEST INFRASTRUCTURE: part of the CPU oracle (see ``oracle/__init__``).
"""
from __future__ import annotations

import numpy as np

# Multipliers and Weyl constants of the paper, for 32- and 64-bit words.
_CONSTS = {
    32: dict(M0=0xD2511F53, M1=0xCD9E8D57, W0=0x9E3779B9, W1=0xBB67AE85),
    64: dict(M0=0xD2E7470EE14C6C93, M1=0xCA5A826395121157,
             W0=0x9E3779B97F4A7C15, W1=0xBB67AE8584CAA73B),
}


def philox_generic(ctr, key, width: int = 32, rounds: int = 10):
    """Reference Philox4x{width}-{rounds} on Python integers (one block).

    ``ctr`` is four words, ``key`` two words; returns the four output words.
    Slow and plain: used to pin the vectorised version and, at width 64,
    to check the round structure against an independent library.
    """
    c = _CONSTS[width]
    mask = (1 << width) - 1
    x0, x1, x2, x3 = (int(v) & mask for v in ctr)
    k0, k1 = (int(v) & mask for v in key)
    for _ in range(rounds):
        p0 = c["M0"] * x0
        p1 = c["M1"] * x2
        hi0, lo0 = (p0 >> width) & mask, p0 & mask
        hi1, lo1 = (p1 >> width) & mask, p1 & mask
        x0, x1, x2, x3 = hi1 ^ x1 ^ k0, lo1, hi0 ^ x3 ^ k1, lo0
        k0 = (k0 + c["W0"]) & mask
        k1 = (k1 + c["W1"]) & mask
    return x0, x1, x2, x3


def philox4x32_10(c0, c1, c2, c3, k0: int, k1: int):
    """Vectorised Philox4x32-10.  Counter words are broadcastable uint32
    arrays; the key is two Python ints.  Returns four uint32 arrays."""
    c = _CONSTS[32]
    M0 = np.uint64(c["M0"])
    M1 = np.uint64(c["M1"])
    lo_mask = np.uint64(0xFFFFFFFF)
    s32 = np.uint64(32)
    x0, x1, x2, x3 = np.broadcast_arrays(
        *(np.asarray(v, dtype=np.uint64) for v in (c0, c1, c2, c3)))
    x0, x1, x2, x3 = (v.copy() for v in (x0, x1, x2, x3))
    ka, kb = int(k0) & 0xFFFFFFFF, int(k1) & 0xFFFFFFFF
    for _ in range(10):
        p0 = M0 * x0
        p1 = M1 * x2
        n0 = (p1 >> s32) ^ x1 ^ np.uint64(ka)
        n1 = p1 & lo_mask
        n2 = (p0 >> s32) ^ x3 ^ np.uint64(kb)
        n3 = p0 & lo_mask
        x0, x1, x2, x3 = n0, n1, n2, n3
        ka = (ka + c["W0"]) & 0xFFFFFFFF
        kb = (kb + c["W1"]) & 0xFFFFFFFF
    return tuple(v.astype(np.uint32) for v in (x0, x1, x2, x3))


def split_seed(seed: int) -> tuple[int, int]:
    """Key words of a 64-bit seed: (low 32 bits, high 32 bits)."""
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    return seed & 0xFFFFFFFF, seed >> 32
