"""Philox4x32-10 in plain numpy (oracle side; test infrastructure only).

Definition: Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as
1, 2, 3" (SC'11), the Philox family with N = 4 words of W = 32 bits and 10
rounds.  One round maps the counter (c0, c1, c2, c3) under the round key
(k0, k1) to

    (hi(M1*c2) ^ c1 ^ k0,  lo(M1*c2),  hi(M0*c0) ^ c3 ^ k1,  lo(M0*c0))

where hi/lo are the upper and lower 32-bit halves of the 64-bit product, and
the key is advanced between rounds by the Weyl increments (W0, W1).  The
multipliers and increments are the published Philox4x32 constants.

Stream convention used by this library (the pages name no generator, so the
mapping is ours): the 64-bit seed gives the key (seed mod 2^32, seed >> 32);
the 4-word block j uses counter (j mod 2^32, j >> 32, 0, 0).  This matches
cuRAND's Philox4_32_10 stream for the same seed, which is what the tests pin
against.
"""

import numpy as np

PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
ROUNDS = 10
_MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(counters, key):
    """Apply the 10-round Philox4x32 bijection.

    counters: uint32 array of shape (n, 4); key: two uint32 words (k0, k1).
    Returns a uint32 array of shape (n, 4).  Arithmetic is done on uint64 so
    that each 32x32-bit product is exact.
    """
    ctr = np.asarray(counters, dtype=np.uint64).reshape(-1, 4)
    c0, c1, c2, c3 = (ctr[:, i].copy() for i in range(4))
    k0 = np.uint64(int(key[0]) & 0xFFFFFFFF)
    k1 = np.uint64(int(key[1]) & 0xFFFFFFFF)
    m0 = np.uint64(PHILOX_M0)
    m1 = np.uint64(PHILOX_M1)
    for r in range(ROUNDS):
        if r > 0:
            k0 = np.uint64((int(k0) + PHILOX_W0) & 0xFFFFFFFF)
            k1 = np.uint64((int(k1) + PHILOX_W1) & 0xFFFFFFFF)
        p0 = m0 * c0
        p1 = m1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return np.stack([c0, c1, c2, c3], axis=1).astype(np.uint32)


def seed_to_key(seed):
    """The 64-bit seed split into the two 32-bit key words (low word first)."""
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    return (seed & 0xFFFFFFFF, seed >> 32)


def block_counters(block_offset, n_blocks):
    """Counters (j mod 2^32, j >> 32, 0, 0) for j = block_offset .. +n_blocks-1."""
    j = np.arange(n_blocks, dtype=np.uint64) + np.uint64(block_offset)
    ctr = np.zeros((n_blocks, 4), dtype=np.uint64)
    ctr[:, 0] = j & _MASK32
    ctr[:, 1] = j >> np.uint64(32)
    return ctr


def philox_u32(seed, block_offset, n_blocks):
    """The raw stream: 4 * n_blocks uint32 words, block by block."""
    out = philox4x32_10(block_counters(block_offset, n_blocks), seed_to_key(seed))
    return out.reshape(-1)
