"""Pins for the oracle's Gaussian noise (Box-Muller from Philox words).

The transform is pinned by its closed-form inverse (the radius gives back
-2 ln u1 and the angle gives back 2 pi u2), by words whose deviates are known
exactly, and by distribution tests that any wrong transform fails.
"""

import numpy as np
import pytest
from scipy import stats

from oracle import noise, philox


def test_u1_one_gives_zero_pair():
    # a = 0xFFFFFFFF -> u1 = ((2^24 - 1) + 1) 2^-24 = 1 -> rho = 0.
    u1, u2 = noise.uniforms_from_words([0xFFFFFFFF], [0x12345678])
    assert u1[0] == 1.0
    ea, eb = noise.box_muller(u1, u2)
    assert ea[0] == 0.0 and eb[0] == 0.0


def test_u2_zero_puts_radius_on_first_slot():
    # b < 256 -> u2 = 0 -> (rho, 0): the cosine goes to the first slot.
    u1, u2 = noise.uniforms_from_words([0x00000000, 0x80000000], [0x000000FF, 0x00000000])
    assert (u2 == 0.0).all()
    ea, eb = noise.box_muller(u1, u2)
    np.testing.assert_allclose(ea, np.sqrt(-2.0 * np.log(u1)), rtol=0, atol=0)
    assert (eb == 0.0).all()
    # a = 0 gives the smallest u1 = 2^-24: rho = sqrt(48 ln 2).
    assert abs(ea[0] - np.sqrt(48.0 * np.log(2.0))) < 1e-14


def test_quarter_turns_are_exact():
    # u2 = 1/4, 1/2, 3/4: the pair is (0, rho), (-rho, 0), (0, -rho) exactly.
    a = [0x7FFFFF00] * 3
    u1, u2 = noise.uniforms_from_words(a, [0x40000000, 0x80000000, 0xC0000000])
    assert u2.tolist() == [0.25, 0.5, 0.75]
    ea, eb = noise.box_muller(u1, u2)
    rho = np.sqrt(-2.0 * np.log(u1[0]))
    assert ea.tolist() == [0.0, -rho, 0.0]
    assert eb.tolist() == [rho, 0.0, -rho]


def test_angle_matches_plain_trig_away_from_quarter_turns():
    rng = np.random.default_rng(1)
    u2 = rng.integers(0, 2**24, size=100000).astype(np.float64) * 2.0 ** -24
    s, c = noise.sincos_pi(2.0 * u2)
    # The plain formula itself is off by up to ~ulp(2 pi) from rounding 2 pi u2.
    np.testing.assert_allclose(s, np.sin(2.0 * np.pi * u2), rtol=0, atol=1e-15)
    np.testing.assert_allclose(c, np.cos(2.0 * np.pi * u2), rtol=0, atol=1e-15)


def test_low_byte_of_words_is_ignored():
    u1a, u2a = noise.uniforms_from_words([0xABCDEF00], [0x13579B00])
    u1b, u2b = noise.uniforms_from_words([0xABCDEFFF], [0x13579BFF])
    assert u1a[0] == u1b[0] and u2a[0] == u2b[0]


def test_uniforms_are_exact_fp32():
    rng = np.random.default_rng(0)
    a = rng.integers(0, 2**32, size=10000, dtype=np.uint64)
    b = rng.integers(0, 2**32, size=10000, dtype=np.uint64)
    u1, u2 = noise.uniforms_from_words(a, b)
    assert (u1.astype(np.float32).astype(np.float64) == u1).all()
    assert (u2.astype(np.float32).astype(np.float64) == u2).all()
    assert (u1 > 0).all() and (u1 <= 1).all() and (u2 >= 0).all() and (u2 < 1).all()


def test_closed_form_inverse_of_the_pair():
    # Radius^2 = -2 ln u1 and angle = 2 pi u2: word a sets the radius, word b the angle.
    words = philox.philox_u32(5, 0, 50000).reshape(-1, 4)
    for p in range(2):
        a, b = words[:, 2 * p], words[:, 2 * p + 1]
        u1, u2 = noise.uniforms_from_words(a, b)
        eps = noise.normal_from_blocks(words.reshape(-1)).reshape(-1, 4)
        ea, eb = eps[:, 2 * p], eps[:, 2 * p + 1]
        np.testing.assert_allclose(ea * ea + eb * eb, -2.0 * np.log(u1), rtol=1e-12, atol=1e-300)
        ang = np.mod(np.arctan2(eb, ea), 2.0 * np.pi)
        ok = ea * ea + eb * eb > 1e-20
        diff = np.abs(ang - 2.0 * np.pi * u2)
        diff = np.minimum(diff, 2.0 * np.pi - diff)
        assert diff[ok].max() < 1e-9


def test_offset_slicing_is_consistent():
    full = noise.normal(9, 0, 103)
    for off in (0, 1, 2, 3, 4, 37, 99):
        np.testing.assert_array_equal(noise.normal(9, off, 103 - off), full[off:])


@pytest.mark.parametrize("seed", [0, 3])
def test_standard_normal_distribution(seed):
    n = 1 << 20
    e = noise.normal(seed, 0, n)
    assert abs(e.mean()) < 5.0 / np.sqrt(n)
    assert abs(e.var() - 1.0) < 5.0 * np.sqrt(2.0 / n)
    assert stats.kstest(e, "norm").pvalue > 1e-4
    # No correlation between neighbours (slot pairs share a radius).
    assert abs(np.corrcoef(e[:-1], e[1:])[0, 1]) < 5.0 / np.sqrt(n)
    # Kurtosis of a normal is 3.
    assert abs(stats.kurtosis(e, fisher=False) - 3.0) < 0.05
