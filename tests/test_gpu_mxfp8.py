"""GPU parity of the MXFP8 quantizer (lg_mx_quantize) with the FP64 oracle:
codes and E8M0 scale bytes bit-exact (integer results of the quantization
decisions), on ragged row counts, every K group size, special blocks
(all-zero, tiny, saturating) and sampled rows of the full-size activations."""

import numpy as np
import pytest
import torch

import lora_gemm_b200 as lg
import synth
from oracle import mxfp8 as omx

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _blocked_offsets(rows_idx, K):
    """Byte offsets of the scales of rows rows_idx (all K blocks) in the blocked layout."""
    kb = np.arange(K // 32)
    r = np.asarray(rows_idx)[:, None]
    g, rr = r // 128, r % 128
    return ((g * (K // 128) + kb[None, :] // 4) * 512 + 16 * (rr % 32) + 4 * (rr // 32) + kb[None, :] % 4)


def _check_rows(x_rows64, codes_rows, scales, rows_idx, K):
    ref_codes, ref_exps = omx.mx_quantize(x_rows64)
    assert np.array_equal(codes_rows, ref_codes), f"{np.count_nonzero(codes_rows != ref_codes)} codes differ"
    got = scales[_blocked_offsets(rows_idx, K)]
    assert np.array_equal(got, (ref_exps + 127).astype(np.uint8))


@pytest.mark.parametrize("rows,K", [(1, 128), (127, 256), (300, 1024), (1000, 3072), (129, 7168)])
def test_quantize_bit_exact(rows, K):
    g = torch.Generator().manual_seed(rows * 13 + K)
    x = torch.randn(rows, K, generator=g) * torch.exp2(torch.randint(-20, 20, (rows, 1), generator=g).float())
    x = x.to(torch.bfloat16)
    if rows > 3:
        x[0, :32] = 0                                   # all-zero block
        x[1, 32:64] = 2.0 ** -130                       # tiny block (exponent clamped at -127)
        x[2, 0] = 480.0                                 # saturates: 480 / 2^0 > 448
        x[3, 64:96] = -(2.0 ** 120)
    codes, scales = lg.mx_quantize(x.to(DEV))
    x64 = x.float().numpy().astype(np.float64)
    sc = scales.cpu().numpy()
    _check_rows(x64, codes.cpu().numpy(), sc, np.arange(rows), K)
    pad = np.arange(rows, (rows + 127) // 128 * 128)
    if pad.size:
        assert (sc[_blocked_offsets(pad, K)] == 0).all()


@pytest.mark.parametrize("name,K", [("2k", 7168), ("2k", 28672)])
def test_quantize_full_size_sampled_rows(name, K):
    w = synth.WORKLOADS[name]
    layer = [i for i, (k, _) in enumerate(w.shapes) if k == K][0]
    x = synth.activations(w, K, layer, DEV)
    codes, scales = lg.mx_quantize(x)
    rows = np.sort(np.random.default_rng(K).choice(w.tokens, 256, replace=False))
    rows = np.unique(np.concatenate([rows, [0, w.tokens - 1]]))
    idx = torch.as_tensor(rows, device=DEV)
    x_rows = x.index_select(0, idx).float().cpu().numpy().astype(np.float64)
    c_rows = codes.index_select(0, idx).cpu().numpy()
    sc = scales.cpu().numpy()
    del x, codes
    torch.cuda.empty_cache()
    _check_rows(x_rows, c_rows, sc, rows, K)


def test_quantize_rejects_bad_shapes():
    x = torch.zeros(4, 96, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(lg.LoraGemmError) as ei:
        lg.mx_quantize(x, scales=torch.empty(1024, dtype=torch.uint8, device=DEV))
    assert ei.value.status == lg.LG_ERR_UNSUPPORTED_SHAPE
