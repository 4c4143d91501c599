"""The synthetic input recipe (synth.py) on the CPU: grid
shapes and token counts of the pages' workloads, per-tensor seeding (the same
seed gives the same draw, different tensors and workloads differ) and the
stated distributions -- x ~ N(0, 1) and W ~ N(0, 1/K) in bf16, A_i ~ N(0, 1/K)
and B_i ~ N(0, 0.01) in FP32 with ranks (384, 128, 64)."""

import math

import pytest
import torch

import synth

CPU = "cpu"


def test_workload_grids_and_token_counts():
    expect = {
        "tiny": ((1, 24, 36, 64), 2304, 1024),
        "768p": ((37, 24, 48, 84), 149184, 3072),
        "1080p": ((37, 24, 68, 120), 301920, 7168),
        "2k": ((37, 24, 90, 160), 532800, 7168),
        "4k": ((37, 24, 136, 240), 1207680, 7168),
    }
    for name, (shape, tokens, d) in expect.items():
        w = synth.WORKLOADS[name]
        assert w.latent_shape == shape and w.tokens == tokens and w.d == d
        assert w.latent_numel == math.prod(shape)
    assert synth.WORKLOADS["2k"].shapes == ((7168, 7168), (7168, 21504), (28672, 7168))
    assert sum(synth.ADAPTER_RANKS) == 576
    assert synth.SIGMA_SCHEDULE == (0.909, 0.857, 0.667, 0.0)
    assert synth.proj_out_shape(synth.WORKLOADS["2k"]) == (7168, 24)
    assert synth.mlp_in_shape(synth.WORKLOADS["2k"]) == (7168, 57344)


def test_draws_are_seeded_per_tensor():
    w = synth.WORKLOADS["tiny"]
    a = synth.activations(w, 1024, 0, CPU, M=64)
    b = synth.activations(w, 1024, 0, CPU, M=64)
    c = synth.activations(w, 1024, 1, CPU, M=64)
    assert torch.equal(a, b) and not torch.equal(a, c)
    other = synth.activations(synth.WORKLOADS["768p"], 1024, 0, CPU, M=64)
    assert not torch.equal(a, other)
    assert not torch.equal(synth.velocity(w, 0, CPU), synth.velocity(w, 1, CPU))


@pytest.mark.parametrize("name", ["tiny"])
def test_distributions(name):
    w = synth.WORKLOADS[name]
    K, N = w.shapes[0]
    x = synth.activations(w, K, 0, CPU).float()
    W = synth.weight(w, 0, CPU).float()
    As, Bs = synth.adapters(w, 0, CPU)
    assert x.dtype == torch.float32 and synth.activations(w, K, 0, CPU).dtype == torch.bfloat16
    assert synth.weight(w, 0, CPU).shape == (N, K)
    assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 1.0) < 0.01
    assert abs(W.std().item() * math.sqrt(K) - 1.0) < 0.01
    assert [A.shape for A in As] == [(r, K) for r in synth.ADAPTER_RANKS]
    assert [B.shape for B in Bs] == [(N, r) for r in synth.ADAPTER_RANKS]
    assert all(A.dtype == torch.float32 and B.dtype == torch.float32 for A, B in zip(As, Bs))
    assert abs(torch.cat([A.flatten() for A in As]).std().item() * math.sqrt(K) - 1.0) < 0.01
    assert abs(torch.cat([B.flatten() for B in Bs]).var().item() - 0.01) < 0.0005
    up = synth.upscaled_latent(w, CPU)
    assert up.shape == w.latent_shape and abs(up.std().item() - 1.0) < 0.01
