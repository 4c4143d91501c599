"""Pins for the oracle's LoRA merge and merged-LoRA linear layer.

* Brute force: pure-Python loops over every index on tiny shapes (a wrong
  transpose, index or dropped term fails here).
* Associativity: the same output through the dense merged delta
  x (W + B_cat A_cat)^T.
* Merge identity: B_cat A_cat = sum_i s_i B_i A_i, and the FP32-stored merged
  factors reproduce the pages' relative merge error (2.2e-8, page
  "Open-H3-Regenerate-2K：MiniMax H3 的开源 4K 精修方案", section
  "三个步如何完成工作") to the same order of magnitude, well under 1e-6.
"""

import json
import math
import os

import numpy as np
import pytest

from oracle import lora

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _brute_merge(As, Bs, scales):
    A_rows, B_rows = [], []
    for A, s in zip(As, scales):
        for r in range(len(A)):
            A_rows.append([s * float(a) for a in A[r]])
    d_out = len(Bs[0])
    for o in range(d_out):
        row = []
        for B in Bs:
            row.extend(float(b) for b in B[o])
        B_rows.append(row)
    return A_rows, B_rows


def _brute_linear(x, W, A_cat, B_cat):
    M, K = len(x), len(x[0])
    N = len(W)
    R = len(A_cat)
    y = [[0.0] * N for _ in range(M)]
    for m in range(M):
        h = [math.fsum(x[m][k] * A_cat[r][k] for k in range(K)) for r in range(R)]
        for n in range(N):
            base = math.fsum(x[m][k] * W[n][k] for k in range(K))
            lo = math.fsum(h[r] * B_cat[n][r] for r in range(R))
            y[m][n] = base + lo
    return y


@pytest.mark.parametrize("ranks,scales", [((2, 1, 3), (0.5, 1.25, -0.75)), ((4,), (1.0,)), ((1, 1), (2.0, 0.0))])
def test_brute_force_tiny(ranks, scales):
    rng = np.random.default_rng(10)
    M, K, N = 3, 5, 4
    As = [rng.standard_normal((r, K)) for r in ranks]
    Bs = [rng.standard_normal((N, r)) for r in ranks]
    x = rng.standard_normal((M, K))
    W = rng.standard_normal((N, K))
    A_cat, B_cat = lora.lora_merge(As, Bs, scales)
    bA, bB = _brute_merge([a.tolist() for a in As], [b.tolist() for b in Bs], scales)
    np.testing.assert_array_equal(A_cat, np.array(bA))
    np.testing.assert_array_equal(B_cat, np.array(bB))
    y = lora.lora_linear(x, W, A_cat, B_cat)
    yb = np.array(_brute_linear(x.tolist(), W.tolist(), bA, bB))
    np.testing.assert_allclose(y, yb, rtol=1e-13, atol=1e-13)


def test_rank_zero_is_plain_gemm_brute_force():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((4, 6))
    W = rng.standard_normal((5, 6))
    y = lora.lora_linear(x, W, np.zeros((0, 6)), np.zeros((5, 0)))
    yb = np.array(_brute_linear(x.tolist(), W.tolist(), [], [[] for _ in range(5)]))
    np.testing.assert_allclose(y, yb, rtol=1e-13, atol=1e-13)


def test_associativity_through_dense_delta():
    rng = np.random.default_rng(12)
    M, K, N = 17, 40, 24
    ranks = (8, 4, 2)
    As = [rng.standard_normal((r, K)) for r in ranks]
    Bs = [rng.standard_normal((N, r)) for r in ranks]
    A_cat, B_cat = lora.lora_merge(As, Bs, (0.5, 1.0, 2.0))
    x = rng.standard_normal((M, K))
    W = rng.standard_normal((N, K))
    y = lora.lora_linear(x, W, A_cat, B_cat)
    y2 = x @ (W + lora.merged_delta(A_cat, B_cat)).T
    np.testing.assert_allclose(y, y2, rtol=1e-12, atol=1e-12)


def test_merge_identity_fp64():
    rng = np.random.default_rng(13)
    d_in, d_out = 48, 40
    ranks = (12, 6, 4)
    scales = (0.7, 1.3, 0.55)
    As = [rng.standard_normal((r, d_in)) for r in ranks]
    Bs = [rng.standard_normal((d_out, r)) for r in ranks]
    A_cat, B_cat = lora.lora_merge(As, Bs, scales)
    assert A_cat.shape == (sum(ranks), d_in) and B_cat.shape == (d_out, sum(ranks))
    d1 = lora.merged_delta(A_cat, B_cat)
    d2 = lora.adapter_delta_sum(As, Bs, scales)
    assert np.linalg.norm(d1 - d2) / np.linalg.norm(d2) < 1e-14


def test_pages_merge_error_figure():
    """FP32-stored merged factors vs the exact sum of the three deltas.

    With the pages' ranks (384, 128, 64) and non-trivial scales, storing
    s_i A_i in FP32 costs one rounding per element (unit roundoff 6e-8), which
    lands the relative error of the merged delta at the pages' order
    (2.2e-8); with unit scales the merge is a copy and the error is 0.
    """
    g = _golden("merge.json")
    ranks = g["adapter_ranks"]
    assert sum(ranks) == g["merged_rank"]
    rng = np.random.default_rng(14)
    d = 256
    As = [(rng.standard_normal((r, d)) / np.sqrt(d)).astype(np.float32) for r in ranks]
    Bs = [(rng.standard_normal((d, r)) * 0.1).astype(np.float32) for r in ranks]
    exact = lora.adapter_delta_sum(As, Bs, (0.7, 1.3, 0.55))
    A_cat, B_cat = lora.lora_merge(As, Bs, (0.7, 1.3, 0.55))
    stored = lora.merged_delta(A_cat.astype(np.float32), B_cat.astype(np.float32))
    rel = np.linalg.norm(stored - exact) / np.linalg.norm(exact)
    assert rel <= 1e-6
    assert 0.1 * g["reported_relative_error"] < rel < 10 * g["reported_relative_error"]
    A1, B1 = lora.lora_merge(As, Bs, (1.0, 1.0, 1.0))
    exact1 = lora.adapter_delta_sum(As, Bs, (1.0, 1.0, 1.0))
    stored1 = lora.merged_delta(A1.astype(np.float32), B1.astype(np.float32))
    assert np.linalg.norm(stored1 - exact1) / np.linalg.norm(exact1) < 1e-15
