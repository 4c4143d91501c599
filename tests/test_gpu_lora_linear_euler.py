"""GPU parity of lora_linear_euler (the step's last projection with the Euler
update and the bf16 copy of the new latent fused into its epilogue) against
the FP64 oracle (oracle.flow.projection_euler_step).

The kernel's velocity is the FP32 accumulator of the bf16 layer, so its error
is the layer's (relative Frobenius <= 1e-2, tests/test_gpu_lora_linear.py);
the update z_new - z_old is held to that bar against (sigma_next - sigma) v
in FP64.  The bf16 copy must equal the round-to-nearest-even bf16 of the
kernel's own FP32 result (PyTorch's conversion) bit for bit.
"""

import numpy as np
import pytest
import torch

import lora_gemm_b200 as lg
import synth
from oracle import flow, lora
from tests.util import rel_fro

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 1e-2
S0, S1 = flow.SCHEDULE[1], flow.SCHEDULE[2]


def _np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _case(F, T, C, K, R, seed):
    g = torch.Generator().manual_seed(seed)
    M = F * T
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    W = (torch.randn(C, K, generator=g) * K ** -0.5).to(torch.bfloat16)
    A = torch.randn(R, K, generator=g) * K ** -0.5
    B = torch.randn(C, R, generator=g) * 0.1
    z = torch.randn(F, C, T, generator=g)
    return x.to(DEV), W.to(DEV), A.to(DEV), B.to(DEV), z.to(DEV)


def _check(x, W, A, B, R, z_old, z_new, zb, T, s0=S0, s1=S1):
    ref = flow.projection_euler_step(_np64(x), _np64(W), _np64(A) if R else np.zeros((0, x.shape[1])),
                                     _np64(B) if R else np.zeros((W.shape[0], 0)), _np64(z_old), T, s0, s1)
    z0 = _np64(z_old)
    assert rel_fro(_np64(z_new) - z0, ref - z0) <= TOL
    if zb is not None:
        assert torch.equal(zb.view(torch.int16), z_new.to(torch.bfloat16).view(torch.int16))


@pytest.mark.parametrize(
    "F,T,C,K,R",
    [
        (1, 256, 24, 128, 0),       # one tile, no LoRA
        (1, 300, 24, 256, 64),      # ragged M
        (3, 100, 16, 512, 576),     # frame boundaries inside tiles and warps, full rank
        (2, 1000, 48, 1024, 576),   # two 16-column loads per warp, the second partly past N
        (1, 640, 8, 128, 64),       # MMA N = 16, 8 columns per warp
        (2, 333, 100, 256, 128),    # > 32 columns per warp: stored 16 at a time
        (1, 512, 300, 256, 64),     # two N tiles (single-SM; one 256-column pair tile)
        (2, 400, 500, 256, 64),     # two N tiles on either variant
        (256, 1, 24, 128, 64),      # one cell per frame: the latent is token-major
        (1, 128, 24, 64, 64),       # smallest K
        (1, 1, 16, 128, 0),         # a single token
    ],
)
@pytest.mark.parametrize("variant", [1, 2])
def test_small_shapes(F, T, C, K, R, variant):
    x, W, A, B, z = _case(F, T, C, K, R, seed=F * T + C + K + R)
    z_old = z.clone()
    zb = torch.empty(z.shape, dtype=torch.bfloat16, device=DEV)
    lg.set_kernel_variant(variant)
    try:
        lg.lora_linear_euler(x, W, A if R else None, B if R else None, z, S0, S1, T, z_bf16=zb)
    finally:
        lg.set_kernel_variant(0)
    assert lg.get_last_device_error() == lg.LG_OK
    _check(x, W, A, B, R, z_old, z, zb, T)


def test_without_bf16_copy_is_identical():
    x, W, A, B, z = _case(2, 700, 24, 512, 576, seed=3)
    z1 = z.clone()
    zb = torch.empty(z.shape, dtype=torch.bfloat16, device=DEV)
    lg.lora_linear_euler(x, W, A, B, z, S0, S1, 700, z_bf16=zb)
    lg.lora_linear_euler(x, W, A, B, z1, S0, S1, 700)
    assert lg.get_last_device_error() == lg.LG_OK
    assert torch.equal(z, z1)


def test_matches_unfused_layer_and_euler_step():
    """With x = I and a bf16-exact velocity the layer is exact, so the fused
    update equals lg.euler_step (FMA in FP32 with the same step) bit for bit,
    and three fused steps from the re-noised latent recover z0 to FP32
    rounding (the closed form of the flow path)."""
    F, T, C = 2, 64, 24
    M = F * T
    g = torch.Generator().manual_seed(11)
    z0 = torch.randn(F, C, T, generator=g).to(torch.bfloat16).float()
    eps = torch.randn(F, C, T, generator=g).to(torch.bfloat16).float()
    vel = eps.double() - z0.double()
    vel_bf = vel.to(torch.bfloat16)                       # what the kernel's W holds
    W = vel_bf.permute(1, 0, 2).reshape(C, M).contiguous().to(DEV)   # W[c, f T + p] = vel[f, c, p]
    x = torch.eye(M, dtype=torch.bfloat16, device=DEV)
    s0 = flow.SCHEDULE[0]
    z = ((1 - s0) * z0.double() + s0 * eps.double()).float().to(DEV)
    z_ref = z.clone()
    v_lat = vel_bf.float().to(DEV)
    for k in range(3):
        lg.lora_linear_euler(x, W, None, None, z, flow.SCHEDULE[k], flow.SCHEDULE[k + 1], T)
        lg.euler_step(z_ref, v_lat, flow.SCHEDULE[k], flow.SCHEDULE[k + 1])
        assert torch.equal(z, z_ref), k
    assert lg.get_last_device_error() == lg.LG_OK
    # vel_bf differs from eps - z0 by its bf16 rounding; the recovered latent
    # is z0 plus that rounding (sigma0 times it), up to FP32 rounding.
    target = z0.double() + s0 * (vel - vel_bf.double())
    assert (z.cpu().double() - target).abs().max().item() <= 1e-5


def test_full_size_2k_sampled_tokens():
    """The 2K latent's last projection (d = 7168 -> 24 channels, rank 576,
    532,800 tokens, 14,400 cells per frame), checked on 256 sampled tokens."""
    w = synth.WORKLOADS["2k"]
    K, C, T = w.d, w.channels, w.height * w.width
    x = synth.activations(w, K, 7, DEV)
    g = torch.Generator(device=DEV).manual_seed(5)
    W = (torch.randn(C, K, device=DEV, generator=g) * K ** -0.5).to(torch.bfloat16)
    As, Bs = [], []
    for r in synth.ADAPTER_RANKS:
        As.append(torch.randn(r, K, device=DEV, generator=g) * K ** -0.5)
        Bs.append(torch.randn(C, r, device=DEV, generator=g) * synth.B_STD)
    A_cat, B_cat = lg.lora_merge(As, Bs, synth.ADAPTER_SCALES)
    z = torch.randn(w.frames, C, T, device=DEV, generator=g)
    z_old = z.clone()
    zb = torch.empty(z.shape, dtype=torch.bfloat16, device=DEV)
    lg.lora_linear_euler(x, W, A_cat, B_cat, z, S0, S1, T, z_bf16=zb)
    assert lg.get_last_device_error() == lg.LG_OK
    assert torch.equal(zb.view(torch.int16), z.to(torch.bfloat16).view(torch.int16))
    rows = np.sort(np.random.default_rng(77).choice(w.tokens, 256, replace=False))
    rows = np.unique(np.concatenate([rows, [0, T - 1, T, w.tokens - 1]]))
    v = lora.lora_linear(_np64(x[torch.as_tensor(rows, device=DEV)]), _np64(W), _np64(A_cat), _np64(B_cat))
    f, p = rows // T, rows % T
    zo = _np64(z_old)[f, :, p]                         # [rows, C]
    zn = _np64(z)[f, :, p]
    assert rel_fro(zn - zo, (S1 - S0) * v) <= TOL


def test_rejects_bad_arguments():
    x, W, A, B, z = _case(1, 256, 24, 128, 64, seed=1)
    with pytest.raises(lg.LoraGemmError) as ei:
        lg.lora_linear_euler(x, W, A, B, z, S0, S1, 100)       # M not a multiple of frame_tokens
    assert ei.value.status == lg.LG_ERR_INVALID_ARG
    with pytest.raises(lg.LoraGemmError) as ei:
        lg.lora_linear_euler(x, W, A, B, z, S0, float("nan"), 256)
    assert ei.value.status == lg.LG_ERR_INVALID_ARG
    zb_over = z.view(-1).view(torch.bfloat16)[: z.numel()]  # a bf16 copy that overlaps z
    with pytest.raises(lg.LoraGemmError) as ei:
        lg.lora_linear_euler(x, W, A, B, z, S0, S1, 256, z_bf16=zb_over)
    assert ei.value.status == lg.LG_ERR_INVALID_ARG
    with pytest.raises(lg.LoraGemmError) as ei:
        lg.lora_linear_euler(x, W, A, B, z, S0, S1, 256, z_bf16=x.view(-1)[: z.numel()])   # copy over x
    assert ei.value.status == lg.LG_ERR_INVALID_ARG


@pytest.mark.parametrize("variant", [1, 2])
def test_wait_timeout_is_reported(variant):
    """A 1 ns wait limit makes the pipeline's waits run out: the status says so
    and the next call with the default limit is correct."""
    x, W, A, B, z = _case(2, 1024, 24, 2048, 576, seed=23)
    lg.set_kernel_variant(variant)
    try:
        lg.set_wait_limit_ns(1)
        try:
            lg.lora_linear_euler(x, W, A, B, z.clone(), S0, S1, 1024)
            status = lg.get_last_device_error()
        finally:
            lg.set_wait_limit_ns(0)
        z_old = z.clone()
        lg.lora_linear_euler(x, W, A, B, z, S0, S1, 1024)
    finally:
        lg.set_kernel_variant(0)
    assert status == lg.LG_ERR_DEVICE_TIMEOUT
    assert lg.get_last_device_error() == lg.LG_OK
    _check(x, W, A, B, 576, z_old, z, None, 1024)
