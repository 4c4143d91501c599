"""GPU parity of lora_linear (tcgen05 kernel) against the FP64 oracle.

Bar: relative Frobenius error <= 1e-2 against y = x W^T + (x A_cat^T) B_cat^T
evaluated in FP64 from the exact input values.  The kernel rounds the merged
factors and h = x A_cat^T to bf16 and y to bf16 (each ~2^-9 relative), so the
expected error is a few 1e-3.  Small shapes compare every element and cover
ragged M and N tails, rank 0 / 64 / 576 and a single K block; the full-size
workloads compare 512 seeded sample rows, with the factors merged by the
oracle from the same adapters.
"""

import numpy as np
import pytest
import torch

import lora_gemm_b200 as lg
import synth
from oracle import lora as olora
from tests.util import rel_fro

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 1e-2


def _np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _rand_layer(M, K, N, R, seed, zero_w=False):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    W = (torch.randn(N, K, generator=g) * K ** -0.5).to(torch.bfloat16)
    if zero_w:
        W.zero_()
    A = torch.randn(R, K, generator=g) * K ** -0.5
    B = torch.randn(N, R, generator=g) * 0.1
    return x.to(DEV), W.to(DEV), A.to(DEV), B.to(DEV)


def _check(x, W, A, B, y):
    ref = olora.lora_linear(_np64(x), _np64(W), _np64(A), _np64(B))
    err = rel_fro(_np64(y), ref)
    assert lg.get_last_device_error() == lg.LG_OK
    return err


@pytest.mark.parametrize(
    "M,K,N,R",
    [
        (128, 64, 224, 0),     # one tile, one K block, no LoRA
        (1, 64, 64, 64),       # single token, N tail inside one tile
        (127, 128, 192, 64),   # M tail
        (300, 256, 448, 128),  # three panels, two full tiles
        (517, 320, 320, 576),  # ragged everything, full rank
        (2304, 1024, 1024, 576),
    ],
)
def test_small_shapes_full_matrix(M, K, N, R):
    x, W, A, B = _rand_layer(M, K, N, R, seed=M * 7 + N)
    y = lg.lora_linear(x, W, A if R else None, B if R else None)
    err = _check(x, W, A, B, y)
    assert err <= TOL, err


@pytest.mark.parametrize("R", [64, 576])
def test_lora_path_alone(R):
    """W = 0: the output is the up-projection of the on-chip h alone."""
    x, W, A, B = _rand_layer(384, 512, 448, R, seed=R, zero_w=True)
    y = lg.lora_linear(x, W, A, B)
    err = _check(x, W, A, B, y)
    assert err <= TOL, err


def test_base_path_alone_many_panels():
    """R = 0 with more panels than SMs (persistent loop) is a plain GEMM."""
    x, W, A, B = _rand_layer(148 * 128 * 2 + 77, 256, 448, 0, seed=3)
    y = lg.lora_linear(x, W, None, None)
    err = _check(x, W, A, B, y)
    assert err <= TOL, err


def test_tiny_workload_full_matrix():
    w = synth.WORKLOADS["tiny"]
    x = synth.activations(w, 1024, 0, DEV)
    W = synth.weight(w, 0, DEV)
    As, Bs = synth.adapters(w, 0, DEV)
    A_cat, B_cat = lg.lora_merge(As, Bs, synth.ADAPTER_SCALES)
    y = lg.lora_linear(x, W, A_cat, B_cat)
    rA, rB = olora.lora_merge([_np64(a) for a in As], [_np64(b) for b in Bs], synth.ADAPTER_SCALES)
    ref = olora.lora_linear(_np64(x), _np64(W), rA, rB)
    err = rel_fro(_np64(y), ref)
    assert lg.get_last_device_error() == lg.LG_OK
    assert err <= TOL, err


def _sampled_rows_case(name, layer, n_rows=512):
    w = synth.WORKLOADS[name]
    K, N = w.shapes[layer]
    x = synth.activations(w, K, layer, DEV)
    W = synth.weight(w, layer, DEV)
    As, Bs = synth.adapters(w, layer, DEV)
    A_cat, B_cat = lg.lora_merge(As, Bs, synth.ADAPTER_SCALES)
    y = lg.lora_linear(x, W, A_cat, B_cat)
    assert lg.get_last_device_error() == lg.LG_OK
    rows = np.sort(np.random.default_rng(w.seed * 10 + layer).choice(w.tokens, n_rows, replace=False))
    rows = np.unique(np.concatenate([rows, [0, w.tokens - 1]]))
    idx = torch.as_tensor(rows, device=DEV)
    y_rows = _np64(y.index_select(0, idx))
    x_rows = _np64(x.index_select(0, idx))
    del x, y
    rA, rB = olora.lora_merge([_np64(a) for a in As], [_np64(b) for b in Bs], synth.ADAPTER_SCALES)
    ref = olora.lora_linear(x_rows, _np64(W), rA, rB)
    torch.cuda.empty_cache()
    return rel_fro(y_rows, ref)


@pytest.mark.parametrize(
    "name,layer",
    [("768p", 0), ("1080p", 0), ("1080p", 1), ("1080p", 2), ("2k", 0), ("2k", 1), ("2k", 2), ("4k", 0), ("4k", 1),
     ("4k", 2)],
)
def test_full_size_sampled_rows(name, layer):
    err = _sampled_rows_case(name, layer)
    assert err <= TOL, err


def test_wait_timeout_is_reported_and_context_survives():
    """A wait limit of 1 ns makes the pipeline's waits run out: the kernel
    records LG_ERR_DEVICE_TIMEOUT, cleans up and returns; the next call with
    the default limit is correct."""
    x, W, A, B = _rand_layer(1024, 1024, 896, 576, seed=9)
    lg.set_wait_limit_ns(1)
    try:
        lg.lora_linear(x, W, A, B)
        status = lg.get_last_device_error()
    finally:
        lg.set_wait_limit_ns(0)
    assert status == lg.LG_ERR_DEVICE_TIMEOUT
    y = lg.lora_linear(x, W, A, B)
    err = _check(x, W, A, B, y)
    assert err <= TOL, err


@pytest.mark.parametrize("variant,G", [(1, 1), (1, 2), (1, 4), (1, 8), (2, 2), (2, 4), (2, 8)])
@pytest.mark.parametrize(
    "M,K,N,R",
    [
        (517, 320, 320, 576),    # ragged M and N, full rank, fewer N tiles than CTAs for G >= 4
        (1000, 1024, 896, 64),   # small rank: slices of 64 / 32 / 16 / 8 ranks
        (300, 256, 1568, 0),     # no LoRA: the cluster only splits N tiles
        (2304, 1024, 1024, 576),
        (37 * 128 + 5, 512, 3584, 576),  # more panels than resident clusters
    ],
)
def test_cluster_sizes(variant, G, M, K, N, R):
    """Every variant and cluster size: CTAs of a cluster share a panel and
    exchange their slices of h; SM pairs split every B tile."""
    x, W, A, B = _rand_layer(M, K, N, R, seed=G * 1000 + M)
    lg.set_kernel_variant(variant)
    lg.set_cluster_size(G)
    try:
        y = lg.lora_linear(x, W, A if R else None, B if R else None)
        err = _check(x, W, A, B, y)
    finally:
        lg.set_cluster_size(0)
        lg.set_kernel_variant(0)
    assert err <= TOL, err


@pytest.mark.parametrize("variant,G", [(1, 4), (2, 2), (2, 4)])
def test_wait_timeout_with_clusters(variant, G):
    x, W, A, B = _rand_layer(2048, 1024, 1792, 576, seed=19)
    lg.set_kernel_variant(variant)
    lg.set_cluster_size(G)
    lg.set_wait_limit_ns(1)
    try:
        lg.lora_linear(x, W, A, B)
        status = lg.get_last_device_error()
    finally:
        lg.set_wait_limit_ns(0)
    try:
        assert status == lg.LG_ERR_DEVICE_TIMEOUT
        y = lg.lora_linear(x, W, A, B)
        err = _check(x, W, A, B, y)
    finally:
        lg.set_cluster_size(0)
        lg.set_kernel_variant(0)
    assert err <= TOL, err


@pytest.mark.parametrize("name,layer", [("768p", 0), ("2k", 0), ("2k", 2)])
def test_full_size_sampled_rows_pair_variant(name, layer):
    lg.set_kernel_variant(2)
    try:
        err = _sampled_rows_case(name, layer)
    finally:
        lg.set_kernel_variant(0)
    assert err <= TOL, err


def test_cluster_size_argument_checked():
    with pytest.raises(lg.LoraGemmError) as ei:
        lg.set_cluster_size(3)
    assert ei.value.status == lg.LG_ERR_INVALID_ARG
    with pytest.raises(lg.LoraGemmError):
        lg.set_cluster_size(16)
    with pytest.raises(lg.LoraGemmError):
        lg.set_kernel_variant(3)


@pytest.mark.parametrize("variant", [1, 2])
@pytest.mark.parametrize("N", [32, 64, 96, 160, 224])
def test_narrow_n_single_tile(variant, N):
    """N below the tile width: one output tile whose MMAs run with N columns
    (an SM pair takes N / 2 B rows from each CTA)."""
    x, W, A, B = _rand_layer(700, 512, N, 576, seed=N + variant)
    lg.set_kernel_variant(variant)
    try:
        y = lg.lora_linear(x, W, A, B)
        err = _check(x, W, A, B, y)
    finally:
        lg.set_kernel_variant(0)
    assert lg.get_last_device_error() == lg.LG_OK
    assert err <= TOL, err


def test_binding_rejects_wrong_output_shapes_before_launch():
    """The binding checks what the C ABI cannot see (output extents, scale
    buffer sizes) and raises before any pointer reaches the library."""
    x, W, A, B = _rand_layer(256, 128, 64, 64, seed=3)
    n0 = lg.launch_count()
    with pytest.raises(ValueError):
        lg.lora_linear(x, W, A, B, y=torch.empty(256, 32, dtype=torch.bfloat16, device=DEV))
    with pytest.raises(ValueError):
        lg.lora_linear_noalloc(x, W, A, B, torch.empty(255, 64, dtype=torch.bfloat16, device=DEV))
    xq, wq = lg.mx_quantize(x), lg.mx_quantize(W)
    n1 = lg.launch_count()
    with pytest.raises(ValueError):
        lg.lora_linear_mxfp8(x, (xq[0], xq[1][:100]), wq, A, B)
    with pytest.raises(ValueError):
        lg.mx_quantize(x, codes=torch.empty(256, 64, dtype=torch.uint8, device=DEV))
    with pytest.raises(ValueError):
        lg.lora_linear_swiglu_mxfp8(x, xq, wq, A, B, out=(torch.empty(256, 64, dtype=torch.uint8, device=DEV),
                                                          torch.empty(16, dtype=torch.uint8, device=DEV)))
    with pytest.raises(ValueError):
        lg.lora_linear(x, W, A, B.cpu())
    assert lg.launch_count() == n1 and n1 - n0 == 2
