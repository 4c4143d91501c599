"""Host emulation of the device Box-Muller arithmetic, checked against
references of higher precision (no GPU, no oracle).

The device evaluates -2 ln u1 by Tang's table method with a Horner-folded
log1p series, sqrt(y) by one third-order step from an FP32 reciprocal square
root seed, and sin/cos(2 pi b 2^-24) from a coarse 1/4096-turn entry and a
fine 2^-24-turn entry combined by the angle-addition formulas (no series).
These tests restate those steps in numpy with the committed tables, every
fused multiply-add evaluated in long double and rounded once to double
(exact up to a 2^-64 relative perturbation before that rounding), and
compare with long-double references on sampled and edge arguments:

* -2 ln u1 within 3 double ulps (relative) for u1 = n 2^-24, n in [1, 2^24];
* sqrt within 2 ulps with the seed moved by the largest error the FP32
  seed can carry (2^-22 relative);
* sin and cos within 4 ulps (relative), exact zeros at the quarter turns.

The bounds the design relies on are a few ulps of double: eps must stay
within ~3e-15 relative for the re-noise to round like the exact value.
"""

import importlib.util
import os

import numpy as np
import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "lora_gemm_b200", "csrc")
LD = np.longdouble
ULP = 2.0**-53  # half the spacing of doubles in [1, 2): relative unit used below

pytestmark = pytest.mark.skipif(np.finfo(np.longdouble).nmant < 63, reason="needs an extended long double")


def _load_gen():
    spec = importlib.util.spec_from_file_location("gen_bm_tables", os.path.join(CSRC, "gen_bm_tables.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


gen = _load_gen()
LOG = np.array(gen.log_table())
COARSE = np.array(gen.trig_coarse_table())
FINE = np.array(gen.trig_fine_table())


def fma(a, b, c):
    return (np.asarray(a, LD) * np.asarray(b, LD) + np.asarray(c, LD)).astype(np.float64)


def neg2_ln_grid24(n):
    """-2 ln(n 2^-24) as the device computes it, for integers n in [1, 2^24]."""
    fb = n.astype(np.float32).view(np.uint32).astype(np.int64)  # exact: n <= 2^24
    frac = fb & 0x7FFFFF
    i = ((frac >> 14) + 1) >> 1
    j = 151 - (fb >> 23) - (i > gen.LOG_SWITCH)
    inv_c, y_tab = LOG[i, 0], LOG[i, 1]
    m = 1.0 + frac.astype(np.float64) * 2.0**-23
    r = fma(m, inv_c, -1.0)
    q = np.full_like(r, 1.0 / 3.0)
    for c in (-2.0 / 5.0, 1.0 / 2.0, -2.0 / 3.0, 1.0, -2.0):
        q = fma(q, r, c)
    base = fma(j.astype(np.float64), 1.3862943611198906188, y_tab)
    return fma(r, q, base)


def sqrt_seeded(y, seed_error):
    """sqrt(y) by the device's third-order step from a seed of the given
    relative error (the FP32 seed's value is replaced by an exact one moved by
    seed_error, then rounded to FP32 as the hardware result is).  Like the
    device, the seed is taken at no less than 2^-24, so y = 0 gives 0."""
    y_seed = np.maximum(y, 2.0**-24).astype(LD)
    r = (1.0 / np.sqrt(y_seed) * LD(1.0 + seed_error)).astype(np.float32).astype(np.float64)
    t = y * r
    h = fma(-t, r, 1.0)
    return fma(t * h, fma(h, 0.375, 0.5), t)


def sincos_turn24(b24):
    """sin and cos of 2 pi b24 2^-24 as the device computes them."""
    w = b24.astype(np.uint64) << np.uint64(8)
    iu = (((w + np.uint64(1 << 19)) & np.uint64(0xFFFFFFFF)) >> np.uint64(20)).astype(np.int64)
    lo = ((w << np.uint64(12)) & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.int32)
    rd = (lo >> 20).astype(np.int64)
    sa, ca = COARSE[iu, 0], COARSE[iu, 1]
    sf = np.where(rd < 0, -FINE[np.abs(rd), 0], FINE[np.abs(rd), 0])
    cf = FINE[np.abs(rd), 1]
    s = fma(sa, cf, ca * sf)
    c = fma(ca, cf, -(sa * sf))
    return s, c


PI_LD = LD("3.14159265358979323846264338327950288")


def _sincos_ref(b24):
    """Long-double sin and cos after exact reduction to the nearest quarter
    turn (|angle| <= pi/4, so the reference keeps its relative accuracy)."""
    nq = (b24 + (1 << 21)) >> 22
    d = b24 - (nq << 22)
    th = LD(2) * PI_LD * d.astype(LD) * LD(2.0) ** -24
    s0, c0 = np.sin(th), np.cos(th)
    q = nq & 3
    return np.choose(q, [s0, c0, -s0, -c0]), np.choose(q, [c0, -s0, -c0, s0])


def _rel_ulps(got, ref):
    ref = np.asarray(ref, LD)
    nz = ref != 0
    return (np.abs((got.astype(LD)[nz] - ref[nz]) / ref[nz]) / LD(ULP)).astype(np.float64)


def _log_args():
    rng = np.random.default_rng(11)
    edges = [1, 2, 3, 2**23 - 1, 2**23, 2**23 + 1, 2**24 - 1, 2**24]
    # 23-bit fractions on both sides of sqrt(2), of the table's switch between
    # entries 106 and 107, and of grid-cell edges, in every binade
    for k in range(0, 24):
        for frac in (0x3504F3, 0x3504F4, 0x353FFF, 0x354000, 0x1FFF, 0x4000, 0x7FC000, 0x7FFFFF):
            n = (1 << k) + ((frac << k) >> 23)
            if 1 <= n <= 2**24:
                edges.append(n)
    return np.unique(np.concatenate([np.array(edges, np.int64), rng.integers(1, 2**24 + 1, 400_000)]))


def test_log_within_three_ulps():
    n = _log_args()
    y = neg2_ln_grid24(n)
    ref = -2.0 * np.log(n.astype(LD) * LD(2.0) ** -24)
    assert np.all(y[ref == 0] == 0.0) and not np.any(np.signbit(y[ref == 0]))
    assert _rel_ulps(y, ref).max() <= 3.0


def test_log_of_one_is_exactly_zero():
    assert neg2_ln_grid24(np.array([2**24], np.int64))[0] == 0.0


@pytest.mark.parametrize("seed_error", [-2.0**-22, 0.0, 2.0**-22])
def test_sqrt_third_order_step_within_two_ulps(seed_error):
    rng = np.random.default_rng(12)
    y = np.concatenate([rng.uniform(2.0**-24, 64.0, 200_000), 2.0 ** rng.uniform(-24, 6, 200_000),
                        [2.0**-24, 1.0, 2.0, 63.999999]])
    s = sqrt_seeded(y, seed_error)
    assert _rel_ulps(s, np.sqrt(y.astype(LD))).max() <= 2.0


def test_sqrt_of_zero_is_zero():
    assert sqrt_seeded(np.array([0.0]), 2.0**-22)[0] == 0.0


def test_two_level_angles_within_four_ulps():
    rng = np.random.default_rng(13)
    quarter = 1 << 22
    edges = []
    for z in (0, quarter, 2 * quarter, 3 * quarter, 4 * quarter):  # zeros of sin or cos
        edges += [z + d for d in range(-5, 6)]
    for iu in (1, 2, 511, 512, 1023, 1024, 2047, 4095):  # split points of the remainder
        edges += [iu * 4096 + d for d in (-2049, -2048, -2047, -1, 0, 1, 2046, 2047, 2048)]
    edges = [e % (1 << 24) for e in edges]
    b24 = np.unique(np.concatenate([np.array(edges, np.int64), rng.integers(0, 1 << 24, 400_000)]))
    s, c = sincos_turn24(b24)
    rs, rc = _sincos_ref(b24)
    for got, ref in ((s, rs), (c, rc)):
        assert np.all(got[np.asarray(ref) == 0] == 0.0)
        assert _rel_ulps(got, ref).max() <= 4.0


def test_exact_values_at_quarter_turns():
    b24 = np.array([0, 1 << 22, 2 << 22, 3 << 22], np.int64)
    s, c = sincos_turn24(b24)
    assert list(s) == [0.0, 1.0, 0.0, -1.0] and list(c) == [1.0, 0.0, -1.0, 0.0]
