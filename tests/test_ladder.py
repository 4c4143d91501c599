"""lg_shift_ladder (host code in the C library) against the oracle's
HyperFlow table and route rule: bit-equal FP32 sigmas for the three IC routes
and across step counts, shifts and starts; argument checks.  No GPU."""

import ctypes
import math

import numpy as np
import pytest

import lora_gemm_b200 as lg
from oracle import flow


@pytest.mark.parametrize("route", ["up3", "up4", "hf8"])
def test_routes_match_oracle(route):
    assert lg.IC_ROUTES[route] == flow.IC_ROUTES_DECIMAL[route]
    assert lg.shift_ladder(lg.IC_ROUTES[route]) == flow.ic_ladder(flow.IC_ROUTES_DECIMAL[route])


@pytest.mark.parametrize("n_steps", [1, 3, 8, 50, 4096])
@pytest.mark.parametrize("shift", [0.5, 1.0, 3.0, 12.0])
def test_sweep_matches_oracle(n_steps, shift):
    rng = np.random.default_rng(n_steps)
    for s0 in [1.0, 0.5, 1e-3] + list(rng.uniform(0.01, 1.0, 5)):
        s0 = float(np.float32(s0))
        assert lg.shift_ladder(s0, n_steps, shift) == flow.ic_ladder(s0, n_steps, shift)


def _raw(sigma0, n_steps, shift, cap):
    buf = (ctypes.c_float * max(cap, 1))()
    n = ctypes.c_int(-7)
    st = lg.lib.lg_shift_ladder(sigma0, n_steps, shift, buf, cap, ctypes.byref(n))
    return st, n.value


@pytest.mark.parametrize(
    "sigma0,n_steps,shift,cap",
    [(0.0, 8, 12.0, 16), (1.5, 8, 12.0, 16), (math.nan, 8, 12.0, 16), (0.5, 0, 12.0, 16), (0.5, 5000, 12.0, 9000),
     (0.5, 8, 0.0, 16), (0.5, 8, -1.0, 16), (0.5, 8, math.inf, 16), (1.0, 8, 12.0, 8)],
)
def test_bad_arguments(sigma0, n_steps, shift, cap):
    st, n = _raw(sigma0, n_steps, shift, cap)
    assert st == lg.LG_ERR_INVALID_ARG and n == -7  # nothing written


def test_exact_capacity():
    st, n = _raw(1.0, 8, 12.0, 9)
    assert st == lg.LG_OK and n == 9
