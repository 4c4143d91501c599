"""The allocation-free entry point lg_lora_linear_noalloc.

It serves callers that cannot allocate device memory when they call the
layer (a plugin in an inference engine whose memory is planned before the
run, a serving loop that must not call cudaMalloc because it synchronizes
the device).  Instead of a caller workspace it uses the library's built-in
scratch array.  This file is collected last so that a run stopping at the
first failure has run everything else first; it passes alone in a fresh
process too, because the first call on the device does the set-up.
"""

import ctypes

import numpy as np
import pytest
import torch

import lora_gemm_b200 as lg
from tests.util import rel_fro

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 1e-2  # the lora_linear parity bar used by the other tests


def _layer(M, K, N, R, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16).to(DEV)
    W = (torch.randn(N, K, generator=g) * K ** -0.5).to(torch.bfloat16).to(DEV)
    A = (torch.randn(R, K, generator=g) * K ** -0.5).to(DEV)
    B = (torch.randn(N, R, generator=g) * 0.1).to(DEV)
    return x, W, A, B


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    # Two different shapes, so the second call would read stale factor copies
    # if it did not overwrite the shared scratch before using it.
    cases = [(1000, 1024, 896, 576, 1), (517, 512, 320, 128, 2)]
    inputs = [_layer(M, K, N, R, s) for M, K, N, R, s in cases]
    refs = [lg.lora_linear(x, W, A, B) for x, W, A, B in inputs]
    outs = [torch.empty_like(r) for r in refs]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for (M, K, N, R, _), (x, W, A, B), y in zip(cases, inputs, outs):
        st = lg.lib.lg_lora_linear_noalloc(
            ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(W.data_ptr()), ctypes.c_void_p(A.data_ptr()),
            ctypes.c_void_p(B.data_ptr()), ctypes.c_void_p(y.data_ptr()), M, K, N, R, stream)
        assert st == lg.LG_OK, lg.status_string(st)
    assert lg.get_last_device_error() == lg.LG_OK
    for ref, y in zip(refs, outs):
        assert rel_fro(_np(y), _np(ref)) <= TOL


def test_noalloc_rejects_shapes_beyond_the_scratch():
    # 2 * 576 * (32768 + 32768) bytes > 48 MiB: refused before anything is read or launched.
    fake = ctypes.c_void_p(0x7F0000000000)
    st = lg.lib.lg_lora_linear_noalloc(fake, fake, fake, fake, ctypes.c_void_p(0x7F1000000000), 128, 32768,
                                       32768, 576, None)
    assert st == lg.LG_ERR_WORKSPACE
