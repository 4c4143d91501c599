"""GPU parity of lora_linear_mxfp8 (block-scaled tcgen05 MMAs for the base
term) against the FP64 MXFP8 oracle.

The oracle quantizes x and W itself (its quantizer is bit-exact with
lg_mx_quantize, tests/test_gpu_mxfp8.py) and evaluates
deq(x) deq(W)^T + (x A_cat^T) B_cat^T in FP64.  The kernel's remaining error
sources are those of the bf16 layer (bf16 factors, bf16 h, bf16 y, FP32
accumulation), so the bar is the same relative Frobenius error of 1e-2.
"""

import numpy as np
import pytest
import torch

import lora_gemm_b200 as lg
import synth
from oracle import lora as olora
from oracle import mxfp8 as omx
from tests.util import rel_fro

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 1e-2


def _np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _layer(M, K, N, R, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    W = (torch.randn(N, K, generator=g) * K ** -0.5).to(torch.bfloat16)
    A = torch.randn(R, K, generator=g) * K ** -0.5
    B = torch.randn(N, R, generator=g) * 0.1
    return x.to(DEV), W.to(DEV), A.to(DEV), B.to(DEV)


def _run(x, W, A, B, R):
    y = lg.lora_linear_mxfp8(x, lg.mx_quantize(x), lg.mx_quantize(W), A if R else None, B if R else None)
    assert lg.get_last_device_error() == lg.LG_OK
    return y


@pytest.mark.parametrize(
    "M,K,N,R",
    [
        (256, 128, 256, 0),      # one tile, one K stage, no LoRA
        (1, 128, 64, 64),        # single token, N tail
        (517, 384, 320, 576),    # ragged M and N, full rank (h partly in shared memory)
        (1000, 1024, 896, 64),
        (2304, 1024, 1024, 576),
    ],
)
def test_small_shapes_full_matrix(M, K, N, R):
    x, W, A, B = _layer(M, K, N, R, seed=M + 3 * K + N)
    y = _run(x, W, A, B, R)
    ref = omx.lora_linear_mxfp8(_np64(x), _np64(W), _np64(A) if R else None, _np64(B) if R else None)
    err = rel_fro(_np64(y), ref)
    assert err <= TOL, err


@pytest.mark.parametrize("G", [2, 4, 8])
def test_cluster_sizes(G):
    M, K, N, R = 37 * 256 + 5, 512, 3584, 576
    x, W, A, B = _layer(M, K, N, R, seed=G)
    lg.set_cluster_size(G)
    try:
        y = _run(x, W, A, B, R)
    finally:
        lg.set_cluster_size(0)
    ref = omx.lora_linear_mxfp8(_np64(x), _np64(W), _np64(A), _np64(B))
    assert rel_fro(_np64(y), ref) <= TOL


def test_quantization_error_against_unquantized_layer():
    """The MXFP8 layer stays close to the bf16 layer's exact value (the
    quantization costs about 1 % on these distributions)."""
    M, K, N, R = 1024, 1024, 1024, 576
    x, W, A, B = _layer(M, K, N, R, seed=5)
    y = _run(x, W, A, B, R)
    exact = olora.lora_linear(_np64(x), _np64(W), _np64(A), _np64(B))
    assert rel_fro(_np64(y), exact) <= 3e-2


@pytest.mark.parametrize("name,layer", [("2k", 0), ("2k", 2)])
def test_full_size_sampled_rows(name, layer):
    w = synth.WORKLOADS[name]
    K, N = w.shapes[layer]
    x = synth.activations(w, K, layer, DEV)
    W = synth.weight(w, layer, DEV)
    As, Bs = synth.adapters(w, layer, DEV)
    A_cat, B_cat = lg.lora_merge(As, Bs, synth.ADAPTER_SCALES)
    y = lg.lora_linear_mxfp8(x, lg.mx_quantize(x), lg.mx_quantize(W), A_cat, B_cat)
    assert lg.get_last_device_error() == lg.LG_OK
    rows = np.sort(np.random.default_rng(w.seed * 10 + layer + 1).choice(w.tokens, 256, replace=False))
    rows = np.unique(np.concatenate([rows, [0, w.tokens - 1]]))
    idx = torch.as_tensor(rows, device=DEV)
    y_rows = _np64(y.index_select(0, idx))
    x_rows = _np64(x.index_select(0, idx))
    del x, y
    torch.cuda.empty_cache()
    ref = omx.lora_linear_mxfp8(x_rows, _np64(W), _np64(A_cat), _np64(B_cat))
    assert rel_fro(y_rows, ref) <= TOL


def test_full_size_d_to_3d_sampled_rows_and_tiles():
    """The 2K grid's d -> 3d layer (7168 -> 21504, the widest N the step
    runs): 258 sampled tokens (first and last included) times 12 of the 84
    output tiles of 256 columns (first and last included); output columns
    depend only on their own W rows, so the oracle takes those rows alone."""
    w = synth.WORKLOADS["2k"]
    layer = 1
    K, N = w.shapes[layer]
    x = synth.activations(w, K, layer, DEV)
    W = synth.weight(w, layer, DEV)
    As, Bs = synth.adapters(w, layer, DEV)
    A_cat, B_cat = lg.lora_merge(As, Bs, synth.ADAPTER_SCALES)
    y = lg.lora_linear_mxfp8(x, lg.mx_quantize(x), lg.mx_quantize(W), A_cat, B_cat)
    assert lg.get_last_device_error() == lg.LG_OK
    rng = np.random.default_rng(w.seed * 10 + layer + 1)
    rows = np.unique(np.concatenate([rng.choice(w.tokens, 256, replace=False), [0, w.tokens - 1]]))
    tiles = np.unique(np.concatenate([rng.choice(N // 256, 10, replace=False), [0, N // 256 - 1]]))
    cols = (tiles[:, None] * 256 + np.arange(256)[None, :]).reshape(-1)
    ridx = torch.as_tensor(rows, device=DEV)
    cidx = torch.as_tensor(cols, device=DEV)
    y_s = _np64(y.index_select(0, ridx).index_select(1, cidx))
    x_rows = _np64(x.index_select(0, ridx))
    W_s = _np64(W.index_select(0, cidx))
    B_s = _np64(B_cat.index_select(0, cidx))
    del x, y
    torch.cuda.empty_cache()
    ref = omx.lora_linear_mxfp8(x_rows, W_s, _np64(A_cat), B_s)
    assert rel_fro(y_s, ref) <= TOL


def test_wait_timeout_is_reported():
    x, W, A, B = _layer(2048, 1024, 1792, 576, seed=19)
    lg.set_wait_limit_ns(1)
    try:
        _ = lg.lora_linear_mxfp8(x, lg.mx_quantize(x), lg.mx_quantize(W), A, B)
        status = lg.get_last_device_error()
    finally:
        lg.set_wait_limit_ns(0)
    assert status == lg.LG_ERR_DEVICE_TIMEOUT
    y = _run(x, W, A, B, 576)
    ref = omx.lora_linear_mxfp8(_np64(x), _np64(W), _np64(A), _np64(B))
    assert rel_fro(_np64(y), ref) <= TOL


def test_rejects_k_not_multiple_of_128():
    x = torch.zeros(8, 192, dtype=torch.bfloat16, device=DEV)
    codes = torch.zeros(8, 192, dtype=torch.uint8, device=DEV)
    sc = torch.zeros(4096, dtype=torch.uint8, device=DEV)
    with pytest.raises(lg.LoraGemmError) as ei:
        lg.lora_linear_mxfp8(x, (codes, sc), (codes, sc), None, None)
    assert ei.value.status == lg.LG_ERR_UNSUPPORTED_SHAPE
