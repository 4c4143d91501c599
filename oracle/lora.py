"""Rank-axis LoRA merge and the merged-LoRA linear layer (oracle side, FP64).

Merge -- page "Open-H3-Regenerate-2K：MiniMax H3 的开源 4K 精修方案"
(comfyui-wiki.com news), section "三个步如何完成工作": three adapters (the
refiner, rank 384; the Turbo adapter, rank 128; the Sharp adapter, rank 64,
in that order) are merged into one file by concatenating their factors along
the rank axis, giving rank 576 on 312 linear layers, stored in FP32; the
merged delta differs from the three separate deltas by 2.2e-8 relative.

With adapter i contributing the delta s_i B_i A_i (A_i: [r_i, d_in],
B_i: [d_out, r_i]), concatenation along the rank axis is

    A_cat = [s_1 A_1; s_2 A_2; s_3 A_3]   (rows)      -> [R, d_in]
    B_cat = [B_1  B_2  B_3]               (columns)   -> [d_out, R]

so that B_cat A_cat = sum_i s_i B_i A_i.  The pages do not say on which
factor the scale sits; this library puts it on A.

Linear layer -- the frozen transformer's linears carry the merged LoRA
("Open-H3-Regenerate-2K: High-Resolution Video Refinement with Few-Step
Diffusion", section "The four-stage refinement pipeline": frozen H3
transformer adapted by the refiner LoRA).  With token activations x: [M, K],
frozen weight W: [N, K] (y = x W^T convention):

    y = x W^T + (x A_cat^T) B_cat^T

The oracle evaluates this in FP64 from the exact input values (the bf16
values of x and W, the FP32 values of A_cat and B_cat) with the unrounded
intermediate h = x A_cat^T.
"""

import numpy as np


def lora_merge(As, Bs, scales):
    """Concatenate adapters along the rank axis.

    Returns (A_cat, B_cat) in FP64.  Each entry of A_cat is the exact product
    s_i * A_i[r, k] of two FP32 numbers (exact in FP64), so its FP32 rounding
    is the correctly rounded merged factor.
    """
    if not (len(As) == len(Bs) == len(scales)):
        raise ValueError("As, Bs and scales must have the same length")
    A_parts = [float(s) * np.asarray(A, dtype=np.float64) for A, s in zip(As, scales)]
    B_parts = [np.asarray(B, dtype=np.float64) for B in Bs]
    for A, B in zip(A_parts, B_parts):
        if A.shape[0] != B.shape[1]:
            raise ValueError("rank mismatch between A_i and B_i")
    return np.concatenate(A_parts, axis=0), np.concatenate(B_parts, axis=1)


def adapter_delta_sum(As, Bs, scales):
    """sum_i s_i B_i A_i in FP64 (the three separate deltas, added)."""
    total = None
    for A, B, s in zip(As, Bs, scales):
        d = float(s) * (np.asarray(B, np.float64) @ np.asarray(A, np.float64))
        total = d if total is None else total + d
    return total


def merged_delta(A_cat, B_cat):
    """B_cat A_cat in FP64: the dense delta that the merged factors encode."""
    return np.asarray(B_cat, np.float64) @ np.asarray(A_cat, np.float64)


def lora_down(x, A_cat):
    """h = x A_cat^T (FP64, unrounded)."""
    return np.asarray(x, np.float64) @ np.asarray(A_cat, np.float64).T


def lora_linear(x, W, A_cat, B_cat):
    """y = x W^T + (x A_cat^T) B_cat^T in FP64.  Rank 0 (empty factors) is allowed."""
    x = np.asarray(x, np.float64)
    y = x @ np.asarray(W, np.float64).T
    A_cat = np.asarray(A_cat, np.float64)
    if A_cat.size:
        y = y + lora_down(x, A_cat) @ np.asarray(B_cat, np.float64).T
    return y
