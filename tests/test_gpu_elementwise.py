"""GPU parity of the HBM-bound kernels against the FP64 oracle.

Tolerances: Philox words bit-exact; eps within 2 FP32 ulp of the oracle's
FP64 value rounded to FP32; re-noise and Euler within 2 ulp of the larger
of the two blended terms (a result that cancels to near zero has no
meaningful ulp of its own); the merge bit-exact (one FP32 rounding of s*A,
an exact copy of B).  Inputs come from synth (torch
generators), never from a kernel under test.
"""

import numpy as np
import pytest
import torch

import lora_gemm_b200 as lg
import synth
from oracle import flow as oflow
from oracle import lora as olora
from oracle import noise as onoise
from oracle import philox as ophilox
from tests.util import rel_fro, ulp_diff, ulp_of

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _f32(a):
    return np.asarray(a, dtype=np.float64).astype(np.float32)


def _blend_bound(a_term, b_term):
    """2 ulp of the larger magnitude of two FP64 terms, as an absolute error bound."""
    big = np.maximum(np.abs(a_term), np.abs(b_term))
    return 2.0 * ulp_of(big)


@pytest.mark.parametrize(
    "seed,block_offset,n_blocks",
    [(0, 0, 1), (3, 0, 7), (1, 12345, 4096), (2**64 - 1, 2**32 - 3, 1000), (4, 0, 28984320 // 4)],
)
def test_philox_u32_bit_exact(seed, block_offset, n_blocks):
    got = lg.philox_u32(n_blocks, seed, block_offset, device=DEV).cpu().numpy().view(np.uint32)
    ref = ophilox.philox_u32(seed, block_offset, n_blocks)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, f"{bad.size} words differ, first at {bad[:5]}"


@pytest.mark.parametrize("n", [1, 2, 3, 5, 8, 1001, 55296])
@pytest.mark.parametrize("offset", [0, 4, 4 * 2**32 + 8])
def test_philox_normal_small(n, offset):
    got = lg.philox_normal(n, 7, offset, device=DEV).cpu().numpy()
    ref = _f32(onoise.normal(7, offset, n))
    d = ulp_diff(got, ref)
    assert d.max() <= 2, f"max ulp {d.max()}"


@pytest.mark.parametrize("name", ["2k", "4k"])
def test_philox_normal_full_latent(name):
    w = synth.WORKLOADS[name]
    n = w.latent_numel
    got = lg.philox_normal(n, w.seed, 0, device=DEV).cpu().numpy()
    ref64 = onoise.normal(w.seed, 0, n)
    d = ulp_diff(got, _f32(ref64))
    hist = np.bincount(np.minimum(d, 3))
    assert d.max() <= 2, f"max ulp {d.max()}, histogram {hist}"
    assert abs(float(got.mean())) < 5 / np.sqrt(n) and abs(float(got.var()) - 1) < 5 * np.sqrt(2 / n)


@pytest.mark.parametrize("name", ["tiny", "768p", "2k", "4k"])
def test_renoise_full_latent(name):
    w = synth.WORKLOADS[name]
    up = synth.upscaled_latent(w, DEV)
    n = up.numel()
    eps = onoise.normal(w.seed, 0, n)
    up_np = up.cpu().numpy().reshape(-1).astype(np.float64)
    for sigma_dec in w.sigma_starts:
        sigma = oflow.as_fp32(sigma_dec)
        got = lg.renoise(up, sigma, w.seed).cpu().numpy().reshape(-1)
        ref = oflow.renoise(up_np, eps, sigma)
        err = np.abs(got.astype(np.float64) - ref)
        bound = _blend_bound((1 - sigma) * up_np, sigma * eps)
        assert (err <= bound).all(), f"sigma {sigma_dec}: worst excess {np.max(err / bound):.3f} x bound"
        assert ulp_diff(got, _f32(ref)).max() <= 2


@pytest.mark.parametrize("n", [1, 3, 4, 6, 13, 4096 + 3])
@pytest.mark.parametrize("sigma", [0.0, 0.001, 0.909, 1.0])
def test_renoise_tails_and_special_sigmas(n, sigma):
    gen = torch.Generator(device="cpu").manual_seed(n)
    up = torch.randn(n, generator=gen).to(DEV)
    sigma32 = oflow.as_fp32(sigma)
    got = lg.renoise(up, sigma32, 11, offset=16).cpu().numpy()
    ref = oflow.renoise(up.cpu().numpy(), onoise.normal(11, 16, n), sigma32)
    assert ulp_diff(got, _f32(ref)).max() <= 2
    if sigma == 0.0:
        assert np.array_equal(got, up.cpu().numpy())


def test_renoise_in_place():
    up = torch.randn(10007, generator=torch.Generator().manual_seed(5)).to(DEV)
    ref = lg.renoise(up, 0.909, 3).clone()
    lg.renoise(up, 0.909, 3, out=up)
    assert torch.equal(up, ref)


@pytest.mark.parametrize("name", ["tiny", "2k", "4k"])
def test_euler_full_latent(name):
    w = synth.WORKLOADS[name]
    x = synth.upscaled_latent(w, DEV)
    x_np = x.cpu().numpy().reshape(-1).astype(np.float64)
    sched = [oflow.as_fp32(s) for s in oflow.SCHEDULE_DECIMAL]
    for k in range(3):
        v = synth.velocity(w, k, DEV)
        v_np = v.cpu().numpy().reshape(-1).astype(np.float64)
        lg.euler_step(x, v, sched[k], sched[k + 1])
        ref = oflow.euler_step(x_np, v_np, sched[k], sched[k + 1])
        got = x.cpu().numpy().reshape(-1)
        err = np.abs(got.astype(np.float64) - ref)
        bound = _blend_bound(x_np, (sched[k + 1] - sched[k]) * v_np)
        assert (err <= bound).all(), f"step {k}: worst excess {np.max(err / bound):.3f}"
        x_np = got.astype(np.float64)  # next step starts from the kernel's FP32 state


@pytest.mark.parametrize("n", [1, 2, 3, 5, 7, 9, 1023])
def test_euler_tails(n):
    g = torch.Generator().manual_seed(n)
    x = torch.randn(n, generator=g).to(DEV)
    v = torch.randn(n, generator=g).to(DEV)
    x0 = x.cpu().numpy().astype(np.float64)
    lg.euler_step(x, v, 0.857, 0.667)
    ref = oflow.euler_step(x0, v.cpu().numpy(), oflow.as_fp32(0.857), oflow.as_fp32(0.667))
    assert ulp_diff(x.cpu().numpy(), _f32(ref)).max() <= 1


@pytest.mark.parametrize("name,start", [("tiny", 0.909), ("2k", 0.909), ("4k", 0.835), ("4k", 0.923)])
def test_refine_chain_recovers_draft(name, start):
    """Re-noise then Euler to 0 with the exact velocity eps - up recovers up (bound 1e-5)."""
    w = synth.WORKLOADS[name]
    up = synth.upscaled_latent(w, DEV)
    eps = lg.philox_normal(up.numel(), w.seed, 0, device=DEV).view_as(up)
    v = eps - up
    sched = [oflow.as_fp32(start)] + [s for s in (oflow.as_fp32(0.857), oflow.as_fp32(0.667), 0.0) if s < oflow.as_fp32(start)]
    x = lg.renoise(up, sched[0], w.seed)
    for k in range(len(sched) - 1):
        lg.euler_step(x, v, sched[k], sched[k + 1])
    err = (x - up).abs().max().item()
    assert err <= 1e-5, err


def _fp32_scales(scales):
    """The scales as the FP32 values the C ABI receives."""
    return tuple(float(np.float32(s)) for s in scales)


@pytest.mark.parametrize("scales", [(1.0, 1.0, 1.0), (0.7, 1.3, 0.55)])
def test_merge_bit_exact_small(scales):
    scales = _fp32_scales(scales)
    w = synth.WORKLOADS["tiny"]
    As, Bs = synth.adapters(w, 0, DEV)
    A_cat, B_cat = lg.lora_merge(As, Bs, scales)
    rA, rB = olora.lora_merge([A.cpu().numpy() for A in As], [B.cpu().numpy() for B in Bs], scales)
    assert np.array_equal(A_cat.cpu().numpy(), rA.astype(np.float32))
    assert np.array_equal(B_cat.cpu().numpy(), rB.astype(np.float32))


@pytest.mark.parametrize("layer", [0, 1, 2])
def test_merge_identity_full_width(layer):
    """B_cat A_cat equals the sum of the three adapter deltas to <= 1e-6 relative (Freivalds probes)."""
    w = synth.WORKLOADS["2k"]
    scales = _fp32_scales((0.7, 1.3, 0.55))
    As, Bs = synth.adapters(w, layer, DEV)
    A_cat, B_cat = lg.lora_merge(As, Bs, scales)
    A64 = A_cat.cpu().numpy().astype(np.float64)
    B64 = B_cat.cpu().numpy().astype(np.float64)
    As_np = [A.cpu().numpy() for A in As]
    Bs_np = [B.cpu().numpy() for B in Bs]
    rA, rB = olora.lora_merge(As_np, Bs_np, scales)
    assert np.array_equal(A_cat.cpu().numpy(), rA.astype(np.float32))
    assert np.array_equal(B_cat.cpu().numpy(), rB.astype(np.float32))
    z = np.random.default_rng(layer).standard_normal((A64.shape[1], 8))
    merged = B64 @ (A64 @ z)
    exact = sum(s * (B.astype(np.float64) @ (A.astype(np.float64) @ z)) for A, B, s in zip(As_np, Bs_np, scales))
    assert rel_fro(merged, exact) <= 1e-6


def test_empty_inputs_launch_nothing():
    before = lg.launch_count()
    e = torch.empty(0, dtype=torch.float32, device=DEV)
    lg.renoise(e, 0.909, 0)
    lg.euler_step(e, e.clone(), 0.909, 0.857)
    lg.philox_normal(0, 0, device=DEV)
    assert lg.launch_count() == before


def test_bad_arguments_raise():
    x = torch.zeros(8, device=DEV)
    with pytest.raises(lg.LoraGemmError) as ei:
        lg.renoise(x, 1.5, 0)
    assert ei.value.status == lg.LG_ERR_INVALID_ARG
    with pytest.raises(lg.LoraGemmError) as ei:
        lg.renoise(x, 0.5, 0, offset=2)
    assert ei.value.status == lg.LG_ERR_INVALID_ARG
    assert lg.get_last_device_error() == lg.LG_OK
