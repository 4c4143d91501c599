"""Seeded synthetic inputs shaped like the pages' latent grids.

This module holds no arithmetic of the method: it only draws the inputs that
both the CUDA path and the FP64 oracle consume (token activations x, frozen
weights W, the three LoRA adapters, the upscaled latent and stand-in
velocities), from torch's own generators, seeded per workload and per
tensor.  No weights or datasets are used: the pages' model and benchmark
clips are not available, so these draws stand in for them.

Workloads (latent [F, C, H, W] with C = 24 channels, one token per latent
cell, so M = F * H * W):

  tiny   1 x 24 x 36 x 64      (2,304 tokens),    d = 1024, seed 0
  768p   37 x 24 x 48 x 84     (149,184 tokens),  d = 3072, seed 1
  1080p  37 x 24 x 68 x 120    (301,920 tokens),  d = 7168, seed 2
  2k     37 x 24 x 90 x 160    (532,800 tokens),  d = 7168, seed 3
  4k     37 x 24 x 136 x 240   (1,207,680 tokens), d = 7168, seed 4

The 2K grid (37 x 24 x 90 x 160, enlarged 2.5x per side from 36 x 64) is the
one printed on "Open-H3-Regenerate-2K: High-Resolution Video Refinement with
Few-Step Diffusion" (sections "From any low-resolution draft to native 4K"
and "Why upscaling happens in latent space"); the 1080P and 4K grids use the
1088- and 2176-row compute grids of "Open-H3-Regenerate-2K-IC" (section
"演示里的 4K 和预设里的 4K，像素并不相同") divided by the VAE's spatial
stride of 16.  The model width d is synthetic (the pages give only 56
attention heads; 7168 = 56 x 128).

Distributions: x ~ N(0, 1) in bf16; W ~ N(0, 1/K) in bf16 (variance over the
fan-in K); adapter i: A_i ~ N(0, 1/K) FP32 [r_i, K], B_i ~ N(0, 0.01) FP32
[N, r_i] (0.01 read as the variance), ranks (384, 128, 64), scales 1.0;
up ~ N(0, 1) FP32; velocities ~ N(0, 1) FP32.
"""

from dataclasses import dataclass, field

import torch

ADAPTER_RANKS = (384, 128, 64)
ADAPTER_SCALES = (1.0, 1.0, 1.0)
B_STD = 0.1  # N(0, 0.01) read as variance 0.01
CHANNELS = 24
SIGMA_SCHEDULE = (0.909, 0.857, 0.667, 0.0)
IC_STARTS = (0.835, 0.923)

# Per-tensor stream ids under one workload seed.
_STREAM_X = 100
_STREAM_W = 200
_STREAM_A = 300
_STREAM_B = 400
_STREAM_UP = 500
_STREAM_V = 600


@dataclass(frozen=True)
class Workload:
    name: str
    frames: int
    height: int
    width: int
    d: int
    seed: int
    shapes: tuple  # (K, N) of each lora_linear layer
    sigma_starts: tuple = field(default=(0.909,))
    channels: int = CHANNELS

    @property
    def tokens(self):
        return self.frames * self.height * self.width

    @property
    def latent_shape(self):
        return (self.frames, self.channels, self.height, self.width)

    @property
    def latent_numel(self):
        return self.frames * self.channels * self.height * self.width


def _three_shapes(d):
    return ((d, d), (d, 3 * d), (4 * d, d))


WORKLOADS = {
    "tiny": Workload("tiny", 1, 36, 64, 1024, 0, ((1024, 1024),)),
    "768p": Workload("768p", 37, 48, 84, 3072, 1, ((3072, 3072),)),
    "1080p": Workload("1080p", 37, 68, 120, 7168, 2, _three_shapes(7168)),
    "2k": Workload("2k", 37, 90, 160, 7168, 3, _three_shapes(7168)),
    "4k": Workload("4k", 37, 136, 240, 7168, 4, _three_shapes(7168), (0.909, 0.835, 0.923)),
}
ORDER = ("tiny", "768p", "1080p", "2k", "4k")


def derive_seed(seed, stream):
    """A distinct 63-bit generator seed per (workload seed, tensor stream)."""
    return (int(seed) * 0x9E3779B97F4A7C15 + int(stream) * 0xBF58476D1CE4E5B9 + 1) % (1 << 63)


def generator(seed, stream, device):
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(derive_seed(seed, stream))
    return g


def fill_normal_(out, std, gen, chunk=1 << 26):
    """out <- cast(std * N(0, 1)) drawn chunk by chunk in FP32 (keeps temporaries small)."""
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        tmp = torch.randn(e - s, generator=gen, device=out.device, dtype=torch.float32)
        if std != 1.0:
            tmp.mul_(std)
        flat[s:e].copy_(tmp)
    return out


def activations(w, K, layer, device, M=None):
    """x ~ N(0, 1), bf16 [M, K] (M defaults to the workload's token count)."""
    M = w.tokens if M is None else M
    x = torch.empty((M, K), dtype=torch.bfloat16, device=device)
    return fill_normal_(x, 1.0, generator(w.seed, _STREAM_X + layer, device))


def weight(w, layer, device, shape=None):
    """W ~ N(0, 1/K), bf16 [N, K]; shape = (K, N) overrides the layer's."""
    K, N = w.shapes[layer] if shape is None else shape
    W = torch.empty((N, K), dtype=torch.bfloat16, device=device)
    return fill_normal_(W, K ** -0.5, generator(w.seed, _STREAM_W + layer, device))


def adapters(w, layer, device, ranks=ADAPTER_RANKS, shape=None):
    """A_i ~ N(0, 1/K) [r_i, K] and B_i ~ N(0, 0.01) [N, r_i], FP32; shape =
    (K, N) overrides the layer's."""
    K, N = w.shapes[layer] if shape is None else shape
    As, Bs = [], []
    for i, r in enumerate(ranks):
        A = torch.empty((r, K), dtype=torch.float32, device=device)
        B = torch.empty((N, r), dtype=torch.float32, device=device)
        fill_normal_(A, K ** -0.5, generator(w.seed, _STREAM_A + 10 * layer + i, device))
        fill_normal_(B, B_STD, generator(w.seed, _STREAM_B + 10 * layer + i, device))
        As.append(A)
        Bs.append(B)
    return As, Bs


# Extra projections around the three layers, drawn on their own streams
# (layer index past the workload's shapes):
#   the step's last projection, d -> C velocity channels per token;
#   the MLP's input projection with SwiGLU, d -> 2 ffn (gate rows, then up
#   rows), ffn = 4 d (the 4d -> d layer's input width).
PROJ_OUT_LAYER = 10
MLP_IN_LAYER = 11


def proj_out_shape(w):
    return (w.d, w.channels)


def mlp_in_shape(w):
    return (w.d, 8 * w.d)


def upscaled_latent(w, device):
    """up ~ N(0, 1), FP32 [F, C, H, W] (stands in for the latent upscaler's output)."""
    up = torch.empty(w.latent_shape, dtype=torch.float32, device=device)
    return fill_normal_(up, 1.0, generator(w.seed, _STREAM_UP, device))


def velocity(w, step, device):
    """A stand-in transformer velocity ~ N(0, 1), FP32 [F, C, H, W]."""
    v = torch.empty(w.latent_shape, dtype=torch.float32, device=device)
    return fill_normal_(v, 1.0, generator(w.seed, _STREAM_V + step, device))
