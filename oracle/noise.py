"""Standard normal noise eps ~ N(0, I) from the Philox stream (oracle side).

The pages draw the re-noise term from standard Gaussian noise ("Three steps
instead of dozens", "Open-H3-Regenerate-2K: High-Resolution Video Refinement
with Few-Step Diffusion") but fix no transform.  This library uses the
textbook Box-Muller transform (Box and Muller, Ann. Math. Statist. 29, 1958):
for independent u1 in (0, 1] and u2 in [0, 1),

    rho = sqrt(-2 ln u1),  eps_a = rho cos(2 pi u2),  eps_b = rho sin(2 pi u2)

are two independent N(0, 1) deviates.

Mapping from the stream (our convention): flat element e (the index in the
[F, C, H, W] latent, plus the caller's offset) belongs to Philox block
j = e // 4 and word slot t = e % 4.  Words (r0, r1) of the block give the
pair for slots 0 and 1, words (r2, r3) the pair for slots 2 and 3.  From a
pair of words (a, b):

    u1 = ((a >> 8) + 1) * 2^-24   in (0, 1]      (never 0, so ln is finite)
    u2 = (b >> 8) * 2^-24         in [0, 1)

Both are exact in FP32.  Slot 0 / 2 takes rho cos(2 pi u2), slot 1 / 3 takes
rho sin(2 pi u2).  The oracle evaluates the transform in FP64 and returns the
unrounded FP64 values; callers round to FP32 where the comparison needs it.

The angle is evaluated as sin/cos of pi t with t = 2 u2 reduced exactly to a
quarter turn plus a remainder |r| <= 1/4 (t is a dyadic rational, so the
reduction has no rounding).  Forming 2 pi u2 first would leave a residue of
order 1e-16 where the exact cosine or sine is 0 (u2 = 1/4, 1/2, 3/4).
"""

import numpy as np

from .philox import philox_u32

TWO_M24 = 2.0 ** -24


def uniforms_from_words(a, b):
    """(u1, u2) in FP64 from two uint32 words; both are exact FP32 values."""
    a = np.asarray(a, dtype=np.uint64)
    b = np.asarray(b, dtype=np.uint64)
    u1 = ((a >> np.uint64(8)) + np.uint64(1)).astype(np.float64) * TWO_M24
    u2 = (b >> np.uint64(8)).astype(np.float64) * TWO_M24
    return u1, u2


def sincos_pi(t):
    """(sin(pi t), cos(pi t)) in FP64 for dyadic t, with exact argument reduction.

    t = n/2 + r with n = round(2t) and |r| <= 1/4 (exact in FP64 for the
    dyadic values used here); the quarter-turn identities
    sin/cos(pi t) = (+-)sin/cos(pi r) then give exact zeros and ones at
    multiples of 1/2 and full relative accuracy elsewhere.
    """
    t = np.asarray(t, dtype=np.float64)
    n = np.rint(2.0 * t)
    r = t - 0.5 * n
    s = np.sin(np.pi * r)
    c = np.cos(np.pi * r)
    q = n.astype(np.int64) & 3
    sin_t = np.select([q == 0, q == 1, q == 2], [s, c, -s], -c)
    cos_t = np.select([q == 0, q == 1, q == 2], [c, -s, -c], s)
    return sin_t, cos_t


def box_muller(u1, u2):
    """The two deviates (rho cos(2 pi u2), rho sin(2 pi u2)) in FP64."""
    rho = np.sqrt(-2.0 * np.log(u1))
    sin_t, cos_t = sincos_pi(2.0 * np.asarray(u2, dtype=np.float64))
    return rho * cos_t, rho * sin_t


def normal_from_blocks(words):
    """Gaussians for whole blocks: words is uint32 (n_blocks*4,) -> FP64 (n_blocks*4,)."""
    w = np.asarray(words, dtype=np.uint32).reshape(-1, 4)
    out = np.empty(w.shape, dtype=np.float64)
    for p in range(2):
        u1, u2 = uniforms_from_words(w[:, 2 * p], w[:, 2 * p + 1])
        ea, eb = box_muller(u1, u2)
        out[:, 2 * p] = ea
        out[:, 2 * p + 1] = eb
    return out.reshape(-1)


def normal(seed, offset, n):
    """eps for flat elements offset .. offset+n-1 (FP64, unrounded).

    offset may be any non-negative integer here; the CUDA entry points ask
    for a multiple of 4 so that blocks line up with 16-byte vectors.
    """
    if n == 0:
        return np.zeros(0, dtype=np.float64)
    first_block = offset // 4
    last_block = (offset + n - 1) // 4
    words = philox_u32(seed, first_block, last_block - first_block + 1)
    eps = normal_from_blocks(words)
    start = offset - 4 * first_block
    return eps[start:start + n]
