"""GPU parity of lora_linear_swiglu_mxfp8 (MXFP8 GEMM with SwiGLU and the
activation quantizer fused into the epilogue) against the FP64 oracle.

The kernel forms silu(gate) * up from its FP32 accumulator and a bf16 h
(the bf16 layer's arithmetic, held to a relative Frobenius error of 1e-2 by
tests/test_gpu_lora_linear.py); the oracle from the exact FP64 layer.  An
element whose pre-quantization values differ by delta lands on the other side
of an E4M3 rounding boundary with probability about delta / step and then
differs by one step (step <= 2^-4 |v| on average over a binade), so the
expected squared difference is about delta * step and the relative Frobenius
difference of the two quantized outputs about sqrt(eps * 2^-4) for a layer
error eps: 0.025 at the layer's bar of 1e-2 (with bf16 h, eps ~ 4e-3, it
measures ~0.015).  Bars: that 0.025 against the oracle's quantized output;
2^-4 (the E4M3 rounding bound) against the unquantized FP64 product; at least
99 % of the scale bytes equal; without LoRA (no bf16 h, eps ~ 1e-8) at least
99 % of the codes equal too."""

import numpy as np
import pytest
import torch

import lora_gemm_b200 as lg
import synth
from oracle import mxfp8 as omx
from tests.util import rel_fro

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _blocked_scales(sc, M, F):
    """[M, F / 32] scale bytes from the blocked layout."""
    r = np.arange(M)[:, None]
    kb = np.arange(F // 32)[None, :]
    off = ((r // 128) * (F // 128) + kb // 4) * 512 + 16 * (r % 128 % 32) + 4 * (r % 128 // 32) + kb % 4
    return sc[off]


def _layer(M, K, F, R, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    W2 = (torch.randn(2 * F, K, generator=g) * K ** -0.5).to(torch.bfloat16)
    A = torch.randn(R, K, generator=g) * K ** -0.5
    B = torch.randn(2 * F, R, generator=g) * 0.1
    return x.to(DEV), W2.to(DEV), A.to(DEV), B.to(DEV)


def _check(x, W2, A, B, R, codes, scales):
    M, F = codes.shape
    s, (ref_codes, ref_exps) = omx.swiglu_mxfp8(_np64(x), _np64(W2), _np64(A) if R else None,
                                                _np64(B) if R else None)
    sc = scales.cpu().numpy()
    got_exps = _blocked_scales(sc, M, F).astype(np.int32) - 127
    got = omx.mx_dequantize(codes.cpu().numpy(), got_exps)
    ref = omx.mx_dequantize(ref_codes, ref_exps)
    assert rel_fro(got, ref) <= (1e-2 * 2.0 ** -4) ** 0.5
    assert rel_fro(got, s) <= 2.0 ** -4
    assert np.mean(got_exps == ref_exps) >= 0.99
    if not R:
        assert np.mean(codes.cpu().numpy() == ref_codes) >= 0.99
    pad = np.arange(M, (M + 127) // 128 * 128)
    if pad.size:
        r = pad[:, None]
        kb = np.arange(F // 32)[None, :]
        off = ((r // 128) * (F // 128) + kb // 4) * 512 + 16 * (r % 128 % 32) + 4 * (r % 128 // 32) + kb % 4
        assert (sc[off] == 0).all()


@pytest.mark.parametrize(
    "M,K,F,R",
    [
        (256, 128, 128, 0),      # one tile, no LoRA
        (1, 128, 128, 0),        # a single token (rows 1-127 of the scale group padded with 0)
        (517, 384, 256, 576),    # ragged M, full rank
        (1000, 1024, 512, 64),
        (2304, 1024, 1024, 576),
    ],
)
def test_swiglu_small_shapes(M, K, F, R):
    x, W2, A, B = _layer(M, K, F, R, seed=M + F)
    codes, scales = lg.lora_linear_swiglu_mxfp8(x, lg.mx_quantize(x), lg.mx_quantize(W2), A if R else None,
                                                B if R else None)
    assert lg.get_last_device_error() == lg.LG_OK
    _check(x, W2, A, B, R, codes, scales)


@pytest.mark.parametrize("G", [2, 4])
def test_swiglu_cluster_sizes(G):
    M, K, F, R = 37 * 256 + 5, 512, 1792, 576
    x, W2, A, B = _layer(M, K, F, R, seed=40 + G)
    lg.set_cluster_size(G)
    try:
        codes, scales = lg.lora_linear_swiglu_mxfp8(x, lg.mx_quantize(x), lg.mx_quantize(W2), A, B)
    finally:
        lg.set_cluster_size(0)
    assert lg.get_last_device_error() == lg.LG_OK
    _check(x, W2, A, B, R, codes, scales)


def test_swiglu_rejects_bad_ffn():
    x = torch.zeros(8, 128, dtype=torch.bfloat16, device=DEV)
    codes = torch.zeros(192, 128, dtype=torch.uint8, device=DEV)   # 2F = 192: F = 96 not a multiple of 128
    sc = torch.zeros(4096, dtype=torch.uint8, device=DEV)
    with pytest.raises(lg.LoraGemmError) as ei:
        lg.lora_linear_swiglu_mxfp8(x, (codes[:8], sc), (codes, sc), None, None,
                                    out=(torch.zeros(8, 96, dtype=torch.uint8, device=DEV), sc))
    assert ei.value.status == lg.LG_ERR_UNSUPPORTED_SHAPE


def test_swiglu_wait_timeout_is_reported():
    M, K, F, R = 2048, 1024, 512, 576
    x, W2, A, B = _layer(M, K, F, R, seed=77)
    xq, wq = lg.mx_quantize(x), lg.mx_quantize(W2)
    lg.set_wait_limit_ns(1)
    try:
        lg.lora_linear_swiglu_mxfp8(x, xq, wq, A, B)
        status = lg.get_last_device_error()
    finally:
        lg.set_wait_limit_ns(0)
    assert status == lg.LG_ERR_DEVICE_TIMEOUT
    codes, scales = lg.lora_linear_swiglu_mxfp8(x, xq, wq, A, B)
    assert lg.get_last_device_error() == lg.LG_OK
    _check(x, W2, A, B, R, codes, scales)


def test_swiglu_at_the_benched_shape_sampled():
    """The shape the step's fused MLP input projection is timed on: a quarter
    of the 2K grid (133,120 tokens), d = 7168 -> 2 x 28,672, merged rank 576,
    drawn as for the timing.  258 sampled tokens (first and last included)
    times 16 of the 224 output tiles of 128 columns (first and last
    included); a tile's outputs depend only on its gate rows and up rows of
    W2 and B_cat, so the oracle takes those rows alone (blocks of 32 along
    the outputs stay whole)."""
    w = synth.WORKLOADS["2k"]
    K, N2 = synth.mlp_in_shape(w)
    F = N2 // 2
    M = (w.tokens // 4) // 128 * 128
    x = synth.activations(w, K, 0, DEV, M=M)
    W2 = synth.weight(w, synth.MLP_IN_LAYER, DEV, shape=(K, N2))
    As, Bs = synth.adapters(w, synth.MLP_IN_LAYER, DEV, shape=(K, N2))
    A_cat, B_cat = lg.lora_merge(As, Bs, synth.ADAPTER_SCALES)
    del As, Bs
    codes, scales = lg.lora_linear_swiglu_mxfp8(x, lg.mx_quantize(x), lg.mx_quantize(W2), A_cat, B_cat)
    assert lg.get_last_device_error() == lg.LG_OK
    rng = np.random.default_rng(17)
    rows = np.unique(np.concatenate([rng.choice(M, 256, replace=False), [0, M - 1]]))
    tiles = np.unique(np.concatenate([rng.choice(F // 128, 14, replace=False), [0, F // 128 - 1]]))
    cols = (tiles[:, None] * 128 + np.arange(128)[None, :]).reshape(-1)
    w_rows = np.concatenate([cols, F + cols])
    ridx = torch.as_tensor(rows, device=DEV)
    got_codes = codes.index_select(0, ridx).index_select(1, torch.as_tensor(cols, device=DEV)).cpu().numpy()
    blocks = (tiles[:, None] * 4 + np.arange(4)[None, :]).reshape(-1)
    r = rows[:, None]
    kb = blocks[None, :]
    off = ((r // 128) * (F // 128) + kb // 4) * 512 + 16 * (r % 128 % 32) + 4 * (r % 128 // 32) + kb % 4
    got_exps = scales.cpu().numpy()[off].astype(np.int32) - 127
    x_rows = _np64(x.index_select(0, ridx))
    widx = torch.as_tensor(w_rows, device=DEV)
    W2_s = _np64(W2.index_select(0, widx))
    B_s = _np64(B_cat.index_select(0, widx))
    del x, W2, codes, scales
    torch.cuda.empty_cache()
    s, (ref_codes, ref_exps) = omx.swiglu_mxfp8(x_rows, W2_s, _np64(A_cat), B_s)
    got = omx.mx_dequantize(got_codes, got_exps)
    ref = omx.mx_dequantize(ref_codes, ref_exps)
    assert rel_fro(got, ref) <= (1e-2 * 2.0 ** -4) ** 0.5
    assert rel_fro(got, s) <= 2.0 ** -4
    assert np.mean(got_exps == ref_exps) >= 0.99
