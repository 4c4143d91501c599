"""The IC sampler routes on the GPU (page "Open-H3-Regenerate-2K-IC",
section "三步接着放大的草稿画，八步从噪声重画"): up3, up4 and hf8 re-noise the
upscaled latent at their start and walk HyperFlow's shift-12 table with
lg_euler_step; the reference row is re-noised at sigma = 0.001.

Each iterate is compared with the oracle's step from the same FP32 input,
within 2 ulp of the larger blended term (and 2 ulp of the oracle's own rounded
re-noise), and with the exact velocity eps - up every route returns the
upscaled latent to 1e-5 (the pages' bound for the three-step check).
"""

import numpy as np
import pytest
import torch

import lora_gemm_b200 as lg
import synth
from oracle import flow as oflow
from oracle import noise as onoise
from tests.util import ulp_diff, ulp_of

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bound(a_term, b_term):
    return 2.0 * ulp_of(np.maximum(np.abs(a_term), np.abs(b_term)))


@pytest.mark.parametrize("route", ["up3", "up4", "hf8"])
@pytest.mark.parametrize("name", ["tiny", "4k"])
def test_route_iterates_match_oracle(name, route):
    w = synth.WORKLOADS[name]
    lad = lg.shift_ladder(lg.IC_ROUTES[route])
    assert lad == oflow.ic_ladder(oflow.IC_ROUTES_DECIMAL[route])
    up = synth.upscaled_latent(w, DEV)
    n = up.numel()
    up_np = up.cpu().numpy().reshape(-1).astype(np.float64)
    eps = onoise.normal(w.seed, 0, n)
    x = lg.renoise(up, lad[0], w.seed)
    got = x.cpu().numpy().reshape(-1)
    ref = oflow.renoise(up_np, eps, lad[0])
    assert (np.abs(got - ref) <= _bound((1 - lad[0]) * up_np, lad[0] * eps)).all()
    assert ulp_diff(got, ref.astype(np.float32)).max() <= 2
    x_np = got.astype(np.float64)
    for k in range(len(lad) - 1):
        v = synth.velocity(w, k, DEV)
        v_np = v.cpu().numpy().reshape(-1).astype(np.float64)
        lg.euler_step(x, v, lad[k], lad[k + 1])
        got = x.cpu().numpy().reshape(-1)
        ref = oflow.euler_step(x_np, v_np, lad[k], lad[k + 1])
        assert (np.abs(got - ref) <= _bound(x_np, (lad[k + 1] - lad[k]) * v_np)).all(), f"step {k}"
        x_np = got.astype(np.float64)
    assert lg.get_last_device_error() == lg.LG_OK


@pytest.mark.parametrize("route", ["up3", "up4", "hf8"])
def test_route_recovers_draft_with_exact_velocity(route):
    w = synth.WORKLOADS["4k"]
    lad = lg.shift_ladder(lg.IC_ROUTES[route])
    up = synth.upscaled_latent(w, DEV)
    eps = lg.philox_normal(up.numel(), w.seed, 0, device=DEV).view_as(up)
    v = eps - up
    x = lg.renoise(up, lad[0], w.seed)
    if route == "hf8":
        assert torch.equal(x, eps)  # sigma 1: pure noise
    for k in range(len(lad) - 1):
        lg.euler_step(x, v, lad[k], lad[k + 1])
    err = (x - up).abs().max().item()
    assert err <= 1e-5, err


@pytest.mark.parametrize("name", ["2k", "4k"])
def test_reference_row_renoise(name):
    """99.9 % draft, 0.1 % noise on a full latent; the reference row draws its
    noise from the slice of the stream after the target's elements."""
    w = synth.WORKLOADS[name]
    sig = oflow.as_fp32(oflow.REFERENCE_ROW_SIGMA_DECIMAL)
    up = synth.upscaled_latent(w, DEV)
    n = up.numel()
    off = (n + 3) // 4 * 4
    got = lg.renoise(up, sig, w.seed, offset=off).cpu().numpy().reshape(-1)
    up_np = up.cpu().numpy().reshape(-1).astype(np.float64)
    eps = onoise.normal(w.seed, off, n)
    ref = oflow.renoise(up_np, eps, sig)
    assert (np.abs(got - ref) <= _bound((1 - sig) * up_np, sig * eps)).all()
    assert ulp_diff(got, ref.astype(np.float32)).max() <= 2
