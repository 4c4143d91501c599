"""Host checks of the constant tables behind the device Box-Muller transform.

The committed include must be exactly what its generator writes, and the
properties the device code relies on must hold: every 1/c_i has at most 28
significant bits (so m * inv_c is exact for a 24-bit mantissa m), it is
within 2^-27 of 1/c_i, the log entries are -2 times the logarithms they
stand for, the coarse angle entries are exact at quarter turns, every angle
entry is on the unit circle and within half a double ulp (relative) of sin
and cos evaluated with 40
decimal digits, also next to the zeros; the two angle tables together give
every 24-bit angle (exhaustively) within a few double ulps.  Pure host work:
no GPU, no oracle.
"""

import importlib.util
import math
import os
import random
import struct
from decimal import Decimal, getcontext
from fractions import Fraction

import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "lora_gemm_b200", "csrc")


def _load_gen():
    spec = importlib.util.spec_from_file_location("gen_bm_tables", os.path.join(CSRC, "gen_bm_tables.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


gen = _load_gen()


def _mantissa_bits_used(x):
    b = struct.unpack("<Q", struct.pack("<d", x))[0] & ((1 << 52) - 1)
    if b == 0:
        return 1
    tz = (b & -b).bit_length() - 1
    return 53 - tz


def test_committed_include_matches_generator():
    with open(os.path.join(CSRC, "lg_bm_tables.inc")) as f:
        assert f.read() == gen.render()


def test_log_table_invariants():
    rows = gen.log_table()
    assert len(rows) == 257
    for i, (inv, y) in enumerate(rows):
        c = 1.0 + i / 256.0
        assert _mantissa_bits_used(inv) <= 28
        assert abs(c * inv - 1.0) <= 2.0**-27
        L = -math.log(2.0 * inv) if i > gen.LOG_SWITCH else -math.log(inv)
        assert y == -2.0 * L  # exactly twice the double nearest the logarithm
        # the stored term never exceeds ln 2 (half of the -2 ln 2 step), so a
        # nonzero multiple of 2 ln 2 always dominates it
        assert abs(y) <= 0.7
        assert math.copysign(1.0, y) > 0 or y != 0.0  # no negative zero
    assert rows[0] == (1.0, 0.0) and rows[256] == (0.5, 0.0)
    # the switch sits at sqrt(2): the entries on either side straddle it
    assert 1 + gen.LOG_SWITCH / 256 < math.sqrt(2) < 1 + (gen.LOG_SWITCH + 1) / 256


def test_log_reduction_is_exact_for_every_mantissa_class():
    """r = m inv_c - 1 is a double exactly (so one fused multiply-add returns
    it unrounded) for 24-bit mantissas m in every table class, including the
    class edges, and |r| stays within 2^-9 + 2^-27."""
    rows = gen.log_table()
    rng = random.Random(0)
    for i in range(257):
        lo = max(1.0, 1.0 + (i - 0.5) / 256.0)
        hi = min(2.0, 1.0 + (i + 0.5) / 256.0)
        ks = [math.ceil(lo * 2**23), math.ceil(hi * 2**23) - 1] + [rng.randrange(math.ceil(lo * 2**23), math.ceil(hi * 2**23)) for _ in range(20)]
        for k in ks:
            m = Fraction(k, 2**23)  # m in [1, 2) with 24 significant bits
            r = m * Fraction(rows[i][0]) - 1
            assert Fraction(float(r)) == r
            assert abs(r) <= Fraction(1, 512) + Fraction(1, 2**27)


_PI40 = Decimal("3.141592653589793238462643383279502884197169")


def _sincos40(i, n):
    """sin and cos of 2 pi i / n by Taylor series with 40 significant digits."""
    getcontext().prec = 45
    a = 2 * _PI40 * i / n
    a = a - (2 * _PI40) * int(a / (2 * _PI40))
    s, c, term_s, term_c = Decimal(0), Decimal(0), a, Decimal(1)
    for k in range(60):
        s += term_s
        c += term_c
        term_s = -term_s * a * a / ((2 * k + 2) * (2 * k + 3))
        term_c = -term_c * a * a / ((2 * k + 1) * (2 * k + 2))
    return s, c


def test_coarse_angle_table_invariants():
    rows = gen.trig_coarse_table()
    n = len(rows)
    assert n == 4096
    exact = {0: (0.0, 1.0), n // 4: (1.0, 0.0), n // 2: (0.0, -1.0), 3 * n // 4: (-1.0, 0.0)}
    for i, (s, c) in enumerate(rows):
        if i in exact:
            assert (s, c) == exact[i]
            assert math.copysign(1.0, s) > 0 or s != 0.0  # no negative zeros
            assert math.copysign(1.0, c) > 0 or c != 0.0
        assert abs(s * s + c * c - 1.0) <= 4e-16
        a = 2 * math.pi * i / n
        assert abs(s - math.sin(a)) <= 1e-15 and abs(c - math.cos(a)) <= 1e-15


def test_fine_angle_table_invariants():
    rows = gen.trig_fine_table()
    assert len(rows) == 2049 and rows[0] == (0.0, 1.0)
    for k, (s, c) in enumerate(rows):
        a = 2 * math.pi * k * 2.0**-24
        assert 0.0 <= s <= a and c <= 1.0  # sin x <= x, cos x <= 1
        assert abs(s - math.sin(a)) <= 1e-18 + 1e-15 * s and abs(c - math.cos(a)) <= 2.3e-16
        assert abs(s * s + c * c - 1.0) <= 4e-16


@pytest.mark.parametrize("i", [1, 2, 511, 512, 513, 1023, 1025, 1535, 2047, 2049, 3000, 3071, 3073, 4094, 4095])
def test_coarse_entries_keep_relative_accuracy_next_to_zeros(i):
    rows = gen.trig_coarse_table()
    s40, c40 = _sincos40(i, len(rows))
    s, c = rows[i]
    assert abs((Decimal(s) - s40) / s40) <= Decimal(1.12e-16)
    assert abs((Decimal(c) - c40) / c40) <= Decimal(1.12e-16)


@pytest.mark.parametrize("k", [1, 2, 3, 100, 1000, 2047, 2048])
def test_fine_entries_correctly_rounded(k):
    s, c = gen.trig_fine_table()[k]
    s40, c40 = _sincos40(k, 2**24)
    assert abs((Decimal(s) - s40) / s40) <= Decimal(1.12e-16)
    assert abs((Decimal(c) - c40) / c40) <= Decimal(1.12e-16)


@pytest.mark.parametrize("i", [1, 37, 1024 + 5, 2048 + 1023, 4095])
def test_coarse_table_symmetry(i):
    rows = gen.trig_coarse_table()
    n = len(rows)
    s, c = rows[i]
    s2, c2 = rows[(i + n // 4) % n]  # a quarter turn later: (c, -s)
    assert (s2, c2) == (c + 0.0, -s + 0.0)


def _two_level_sincos(b24):
    """The device's angle split, in exact rational arithmetic on the table
    entries, with each product and fused sum rounded to double as the device
    rounds them: w = b24 << 8, iu = (w + 2^19) >> 20 mod 4096, rd = the low 12
    bits of b24 as a signed integer."""
    coarse, fine = gen.trig_coarse_table(), gen.trig_fine_table()
    iu = ((b24 + 2048) >> 12) % 4096
    rd = ((b24 & 4095) ^ 2048) - 2048
    sa, ca = coarse[iu]
    sb, cb = fine[abs(rd)]
    sb = -sb if rd < 0 else sb
    s = float(Fraction(sa) * Fraction(cb) + Fraction(ca * sb))
    c = float(Fraction(ca) * Fraction(cb) - Fraction(sa * sb))
    return s, c


@pytest.mark.parametrize("b24", [0, 1, 2047, 2048, 2049, 4095, 4096, 4097, (1 << 22) - 2049, (1 << 22) - 2048,
                                 (1 << 22) - 1, 1 << 22, (1 << 22) + 2047, (1 << 23) - 1, 1 << 23, (1 << 23) + 1,
                                 (3 << 22) - 1, 3 << 22, (1 << 24) - 2049, (1 << 24) - 2048, (1 << 24) - 1,
                                 0x5A5A5A, 0x123456, 0xABCDEF])
def test_two_level_angles_near_zeros_and_splits(b24):
    """Next to the zeros of sin and cos, at the split points of the remainder
    and at the wrap of the coarse index, the two lookups give sin and cos of
    2 pi b24 2^-24 within 4 double ulps (relative)."""
    s, c = _two_level_sincos(b24)
    s40, c40 = _sincos40(b24, 2**24)
    for got, ref in ((s, s40), (c, c40)):
        if abs(ref) < Decimal("1e-30"):  # an exact zero (the 40-digit series leaves ~1e-43)
            assert got == 0.0
        else:
            assert abs((Decimal(got) - ref) / ref) <= Decimal(4 * 2.0**-53)
