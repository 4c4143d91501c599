"""Pin the oracle's Philox4x32-10 to an independent implementation.

The pin is cuRAND's host-side Philox4_32_10 generator (a library run on the
CPU; no GPU involved).  cuRAND keys the generator with the 64-bit seed and
interleaves 65536 subsequences: the 4-word output block b (b = word offset /
4, set with curandSetGeneratorOffset) is Philox applied to the counter
(k mod 2^32, k >> 32, t, 0) with k = b // 65536 and t = b % 65536.  Agreement
for several keys (including ones with a non-zero high word) and offsets
(including k past 2^32) pins the round function, the constants and the key
schedule; the t = 0 blocks are exactly this library's stream, counter
(j mod 2^32, j >> 32, 0, 0), which pins the (seed, block) mapping too.
"""

import ctypes
import glob
import os

import numpy as np
import pytest

from oracle import philox

CURAND_RNG_PSEUDO_PHILOX4_32_10 = 161


def _load_curand():
    cands = ["/usr/local/cuda/lib64/libcurand.so.10", "libcurand.so.10", "libcurand.so"]
    try:
        import nvidia  # type: ignore

        for base in nvidia.__path__:
            cands += glob.glob(os.path.join(base, "curand", "lib", "libcurand.so*"))
    except Exception:
        pass
    for c in cands:
        try:
            return ctypes.CDLL(c)
        except OSError:
            continue
    return None


_CURAND = _load_curand()
needs_curand = pytest.mark.skipif(_CURAND is None, reason="libcurand not found on this host")


def curand_host_stream(seed, word_offset, n_words):
    lib = _CURAND
    gen = ctypes.c_void_p()
    assert lib.curandCreateGeneratorHost(ctypes.byref(gen), CURAND_RNG_PSEUDO_PHILOX4_32_10) == 0
    try:
        assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
        assert lib.curandSetGeneratorOffset(gen, ctypes.c_ulonglong(word_offset)) == 0
        out = np.zeros(n_words, dtype=np.uint32)
        assert lib.curandGenerate(gen, out.ctypes.data_as(ctypes.c_void_p), ctypes.c_size_t(n_words)) == 0
    finally:
        lib.curandDestroyGenerator(gen)
    return out


CURAND_SUBSEQUENCES = 65536


def curand_block_counters(block_offset, n_blocks):
    """Counters cuRAND's host generator uses for output blocks b0 .. b0+n-1."""
    b = np.arange(n_blocks, dtype=np.uint64) + np.uint64(block_offset)
    k = b // np.uint64(CURAND_SUBSEQUENCES)
    t = b % np.uint64(CURAND_SUBSEQUENCES)
    ctr = np.zeros((n_blocks, 4), dtype=np.uint64)
    ctr[:, 0] = k & np.uint64(0xFFFFFFFF)
    ctr[:, 1] = k >> np.uint64(32)
    ctr[:, 2] = t
    return ctr


@needs_curand
@pytest.mark.parametrize("seed", [0, 1, 3, 4, 0x0123456789ABCDEF, 2**64 - 1])
@pytest.mark.parametrize("block_offset", [0, 65530, 1000003 * 65536 + 17, (2**32 + 5) * 65536 - 9])
def test_philox_bijection_matches_curand_host(seed, block_offset):
    n_blocks = 4096
    ours = philox.philox4x32_10(curand_block_counters(block_offset, n_blocks), philox.seed_to_key(seed))
    ref = curand_host_stream(seed, 4 * block_offset, 4 * n_blocks).reshape(-1, 4)
    np.testing.assert_array_equal(ours, ref)


@needs_curand
@pytest.mark.parametrize("seed", [0, 3, 2**64 - 1])
@pytest.mark.parametrize("j", [0, 1, 12345, 2**32 - 1, 2**32 + 3])
def test_library_stream_is_curand_subsequence_zero(seed, j):
    # Block j of this library's stream is cuRAND's block (k = j, t = 0).
    ours = philox.philox_u32(seed, j, 1)
    ref = curand_host_stream(seed, 4 * CURAND_SUBSEQUENCES * j, 4)
    np.testing.assert_array_equal(ours, ref)


def test_philox_is_a_bijection_on_a_sample():
    # Distinct counters under one key must give distinct outputs.
    out = philox.philox_u32(11, 0, 1 << 16).reshape(-1, 4)
    as_int = (out[:, 0].astype(np.uint64) << np.uint64(32)) | out[:, 1].astype(np.uint64)
    assert len(np.unique(as_int)) == len(as_int)


def test_seed_and_counter_split():
    assert philox.seed_to_key(0x0123456789ABCDEF) == (0x89ABCDEF, 0x01234567)
    ctr = philox.block_counters(2**32 + 5, 2)
    assert ctr[0].tolist() == [5, 1, 0, 0]
    assert ctr[1].tolist() == [6, 1, 0, 0]
