"""Pins for the oracle's re-noise and Euler steps.

The pins come from the flow-matching construction on "Open-H3-Regenerate-2K:
High-Resolution Video Refinement with Few-Step Diffusion": along the linear
path z_sigma = (1 - sigma) z0 + sigma eps the exact velocity is v = eps - z0,
so an Euler step from sigma to sigma' lands exactly on z_sigma', and any
schedule that ends at 0 returns z0 (section "Training: learn what degradation
removed" for the path, section "Three steps instead of dozens" for the
re-noise and the schedule).
"""

import json
import os

import numpy as np
import pytest

from oracle import flow

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_schedule_constants_match_pages():
    g = _golden("schedule.json")
    assert list(flow.SCHEDULE_DECIMAL) == g["sigma_schedule"]
    assert list(flow.IC_STARTS_DECIMAL) == g["ic_starts"]
    assert flow.SIGMA0 == float(np.float32(g["sigma0"]))
    assert flow.SCHEDULE[-1] == 0.0


def test_schedule_coefficients_exact_in_fp32():
    # Sterbenz: for y/2 <= x <= 2y, x - y is exact.  The kernels compute
    # 1 - sigma and sigma_next - sigma in FP32; they must equal the exact
    # differences the oracle uses.
    sig = [np.float32(s) for s in flow.SCHEDULE_DECIMAL]
    for s in sig + [np.float32(s) for s in flow.IC_STARTS_DECIMAL]:
        assert float(np.float32(1.0) - s) == 1.0 - float(s)
    for a, b in zip(sig[:-1], sig[1:]):
        assert float(b - a) == float(b) - float(a)


@pytest.mark.parametrize("start", [0.909, 0.835, 0.923])
def test_exact_velocity_recovers_z0(start):
    rng = np.random.default_rng(1)
    z0 = rng.standard_normal(10000)
    eps = rng.standard_normal(10000)
    sched = [flow.as_fp32(start)] + [s for s in flow.SCHEDULE[1:]]
    if start != 0.909:
        sched = [flow.as_fp32(start), 0.0]
    zs = flow.refine(z0, eps, sched, lambda z, k: flow.exact_velocity(z0, eps))
    # Every iterate sits on the flow path ...
    for z, s in zip(zs, sched):
        np.testing.assert_allclose(z, flow.flow_point(z0, eps, s), rtol=0, atol=1e-14)
    # ... and the last one is z0 (the pages' bound for this check is 1e-5).
    assert np.abs(zs[-1] - z0).max() < 1e-14


def test_three_step_schedule_recovers_z0():
    rng = np.random.default_rng(2)
    z0 = rng.standard_normal(5000)
    eps = rng.standard_normal(5000)
    zs = flow.refine(z0, eps, flow.SCHEDULE, lambda z, k: flow.exact_velocity(z0, eps))
    assert len(zs) == 4
    assert np.abs(zs[-1] - z0).max() < 1e-14


def test_renoise_special_cases():
    rng = np.random.default_rng(3)
    up = rng.standard_normal(100)
    eps = rng.standard_normal(100)
    np.testing.assert_array_equal(flow.renoise(up, eps, 0.0), up)
    np.testing.assert_array_equal(flow.renoise(up, eps, 1.0), eps)
    # sigma0 = 0.909 keeps 9.1 % of the draft.
    x = flow.renoise(up, np.zeros(100), flow.SIGMA0)
    np.testing.assert_allclose(x, (1.0 - flow.SIGMA0) * up, rtol=1e-15)


def test_euler_special_cases():
    rng = np.random.default_rng(4)
    x = rng.standard_normal(100)
    v = rng.standard_normal(100)
    np.testing.assert_array_equal(flow.euler_step(x, v, 0.5, 0.5), x)
    # Stepping to sigma' = sigma - 1 adds v with a minus sign.
    np.testing.assert_allclose(flow.euler_step(x, v, 1.0, 0.0), x - v, rtol=0, atol=1e-15)


# --- HyperFlow table and the IC routes ("三步接着放大的草稿画，八步从噪声重画") ---


def test_hyperflow_constants_match_page():
    g = _golden("schedule.json")["hyperflow"]
    assert flow.HYPERFLOW_STEPS == g["steps"] and flow.HYPERFLOW_SHIFT == g["video_shift"]
    assert {r: v["sigma0"] for r, v in g["routes"].items()} == flow.IC_ROUTES_DECIMAL
    assert flow.REFERENCE_ROW_SIGMA_DECIMAL == g["reference_row_sigma"]


@pytest.mark.parametrize("route", ["up3", "up4", "hf8"])
def test_route_step_counts_match_page(route):
    """The page counts three steps for up3, one more for up4 and eight for hf8."""
    g = _golden("schedule.json")["hyperflow"]["routes"][route]
    lad = flow.ic_ladder(g["sigma0"])
    assert len(lad) - 1 == g["steps"]
    assert lad[0] == flow.as_fp32(g["sigma0"]) and lad[-1] == 0.0
    assert all(a > b for a, b in zip(lad, lad[1:]))


def test_hyperflow_table_properties():
    tab = flow.hyperflow_table()
    assert len(tab) == 9 and tab[0] == 1.0 and tab[-1] == 0.0  # hf8 starts from pure noise
    # the printed up4 start is the table point at t = 1/2, to the printed digits
    assert round(tab[4], 3) == 0.923
    # inverting the shift, t = sigma / (s - (s - 1) sigma), gives back the uniform grid
    s = flow.HYPERFLOW_SHIFT
    for k, sig in enumerate(tab):
        assert abs(sig / (s - (s - 1) * sig) - (1 - k / 8)) < 1e-15
    # shift 1 is the unshifted grid; a larger shift pushes every interior point up
    assert flow.hyperflow_table(shift=1.0) == [1 - k / 8 for k in range(9)]
    for a, b in zip(flow.hyperflow_table(shift=3.0)[1:-1], tab[1:-1]):
        assert a < b


def test_route_coefficients_exact_in_fp32():
    """Sterbenz again: every dt of every route and 1 - sigma0 (sigma0 >= 1/2)
    are exact in FP32, so the kernels' coefficients equal the oracle's."""
    for start in flow.IC_ROUTES_DECIMAL.values():
        lad = [np.float32(x) for x in flow.ic_ladder(start)]
        assert float(np.float32(1.0) - lad[0]) == 1.0 - float(lad[0])
        for a, b in zip(lad[:-1], lad[1:]):
            assert float(b - a) == float(b) - float(a)


@pytest.mark.parametrize("route", ["up3", "up4", "hf8"])
def test_routes_recover_z0_with_exact_velocity(route):
    rng = np.random.default_rng(7)
    z0 = rng.standard_normal(5000)
    eps = rng.standard_normal(5000)
    lad = flow.ic_ladder(flow.IC_ROUTES_DECIMAL[route])
    zs = flow.refine(z0, eps, lad, lambda z, k: flow.exact_velocity(z0, eps))
    for z, sig in zip(zs, lad):
        np.testing.assert_allclose(z, flow.flow_point(z0, eps, sig), rtol=0, atol=1e-14)
    if route == "hf8":
        assert np.array_equal(zs[0], eps)  # sigma 1: the draft does not enter the start
    assert np.abs(zs[-1] - z0).max() < 1e-14


def test_reference_row_blend():
    """99.9 % draft, 0.1 % noise: the FP32 sigma is within 2^-34 of 0.001 and
    the blend is the exact convex combination."""
    sig = flow.as_fp32(flow.REFERENCE_ROW_SIGMA_DECIMAL)
    assert abs(sig - 0.001) < 2.0**-34
    up = np.array([1.0, -2.0, 0.0])
    eps = np.array([0.0, 1.0, 5.0])
    np.testing.assert_array_equal(flow.renoise(up, eps, sig), (1 - sig) * up + sig * eps)


def test_projection_euler_brute_force_tiny():
    """The fused projection + Euler oracle against explicit loops over the
    latent's flat index ((f C + c) T + p), with a rank-2 LoRA."""
    rng = np.random.default_rng(31)
    F, C, T, K, R = 2, 3, 5, 8, 2
    M = F * T
    x = rng.standard_normal((M, K))
    W = rng.standard_normal((C, K))
    A = rng.standard_normal((R, K))
    B = rng.standard_normal((C, R))
    z = rng.standard_normal(F * C * T)
    s0, s1 = flow.SCHEDULE[1], flow.SCHEDULE[2]
    got = flow.projection_euler_step(x, W, A, B, z, T, s0, s1)
    for f in range(F):
        for c in range(C):
            for p in range(T):
                m = f * T + p
                v = sum(x[m, k] * W[c, k] for k in range(K))
                v += sum(sum(x[m, k] * A[r, k] for k in range(K)) * B[c, r] for r in range(R))
                i = (f * C + c) * T + p
                assert abs(got[i] - (z[i] + (s1 - s0) * v)) <= 1e-12 * (1 + abs(z[i]) + abs(v))


def test_projection_euler_recovers_z0():
    """With x = I (one token per row of W) and W holding eps - z0 in token
    order, three fused steps from the re-noised latent land on z0 -- the
    closed form of the flow path -- only if tokens map to the right cells."""
    rng = np.random.default_rng(32)
    F, C, T = 3, 4, 6
    M = F * T
    z0 = rng.standard_normal((F, C, T))
    eps = rng.standard_normal((F, C, T))
    vel = (eps - z0).transpose(0, 2, 1).reshape(M, C)  # token-major velocity
    x = np.eye(M)
    W = vel.T
    z = flow.renoise(z0, eps, flow.SCHEDULE[0])
    for k in range(3):
        z = flow.projection_euler_step(x, W, np.zeros((0, M)), np.zeros((C, 0)), z, T, flow.SCHEDULE[k],
                                       flow.SCHEDULE[k + 1])
    assert np.allclose(z, z0, rtol=0, atol=1e-14)
    # The token-major layout read as channel-major misses.
    wrong = flow.euler_step(flow.renoise(z0, eps, flow.SCHEDULE[0]), vel.reshape(F, C, T), flow.SCHEDULE[0], 0.0)
    assert not np.allclose(wrong, z0, atol=1e-3)


def test_projection_euler_zero_step_keeps_z():
    rng = np.random.default_rng(33)
    x = rng.standard_normal((8, 16))
    W = rng.standard_normal((2, 16))
    z = rng.standard_normal((2, 2, 4))
    assert np.array_equal(flow.projection_euler_step(x, W, np.zeros((0, 16)), np.zeros((2, 0)), z, 4, 0.5, 0.5), z)
