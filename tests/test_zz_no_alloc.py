"""The allocation-free entry point lg_lora_linear_noalloc.

It serves callers that cannot allocate device memory when they call the
layer (a plugin in an inference engine whose memory is planned before the
run, a serving loop that must not call cudaMalloc because it synchronizes
the device).  Instead of a caller workspace it uses the library's built-in
scratch array.  It runs the very kernels of lg_lora_linear with the same
launch configuration, so its output must equal lg_lora_linear's bit for bit.

This file is collected last so that a run stopping at the first failure has
run everything else first; it passes alone in a fresh process too, because
the first call on the device does the set-up.
"""

import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import lora_gemm_b200 as lg
from oracle import lora as olora
from tests.util import rel_fro

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 1e-2  # the lora_linear parity bar against the FP64 oracle
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _layer(M, K, N, R, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16).to(DEV)
    W = (torch.randn(N, K, generator=g) * K ** -0.5).to(torch.bfloat16).to(DEV)
    A = (torch.randn(R, K, generator=g) * K ** -0.5).to(DEV)
    B = (torch.randn(N, R, generator=g) * 0.1).to(DEV)
    return x, W, A, B


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


def _call_noalloc(x, W, A, B, y, M, K, N, R):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lg.lib.lg_lora_linear_noalloc(
        ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(W.data_ptr()),
        ctypes.c_void_p(A.data_ptr()) if R else None, ctypes.c_void_p(B.data_ptr()) if R else None,
        ctypes.c_void_p(y.data_ptr()), M, K, N, R, stream)


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    # Two different shapes, the second with a smaller rank, so the second call
    # would read stale factor copies if it did not overwrite the shared
    # scratch before using it.
    cases = [(1000, 1024, 896, 576, 1), (517, 512, 320, 128, 2)]
    inputs = [_layer(M, K, N, R, s) for M, K, N, R, s in cases]
    refs = [lg.lora_linear(x, W, A, B) for x, W, A, B in inputs]
    outs = [torch.full_like(r, float("nan")) for r in refs]
    for (M, K, N, R, _), (x, W, A, B), y in zip(cases, inputs, outs):
        st = _call_noalloc(x, W, A, B, y, M, K, N, R)
        assert st == lg.LG_OK, lg.status_string(st)
    assert lg.get_last_device_error() == lg.LG_OK
    for ref, y in zip(refs, outs):
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))


def test_noalloc_near_the_scratch_limit():
    """The 2K grid's 4d -> d layer (28672 -> 7168, rank 576): 41.3 MB of
    factor copies, most of the 48 MiB array; ragged M."""
    M, K, N, R = 300, 28672, 7168, 576
    need = lg.lora_linear_workspace_size(M, K, N, R)
    assert 40e6 < need <= lg.LG_NOALLOC_SCRATCH_BYTES
    x, W, A, B = _layer(M, K, N, R, 3)
    ref = lg.lora_linear(x, W, A, B)
    y = torch.full_like(ref, float("nan"))
    for _ in range(2):
        y.fill_(float("nan"))
        st = _call_noalloc(x, W, A, B, y, M, K, N, R)
        assert st == lg.LG_OK, lg.status_string(st)
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
    rows = np.arange(0, M, 37)
    exact = olora.lora_linear(_np(x[rows]), _np(W), _np(A), _np(B))
    assert rel_fro(_np(y[rows]), exact) <= TOL


@pytest.mark.parametrize("M,K,N,R", [(257, 256, 448, 576), (131, 128, 192, 0)])
def test_noalloc_binding_against_the_oracle(M, K, N, R):
    """The Python binding's lora_linear_noalloc against the FP64 oracle,
    rank 576 and rank 0 (no scratch needed)."""
    x, W, A, B = _layer(M, K, N, R, M + R)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    lg.lora_linear_noalloc(x, W, A if R else None, B if R else None, y)
    assert lg.get_last_device_error() == lg.LG_OK
    exact = olora.lora_linear(_np(x), _np(W), _np(A), _np(B))
    assert rel_fro(_np(y), exact) <= TOL
    ref = lg.lora_linear(x, W, A if R else None, B if R else None)
    assert torch.equal(y.view(torch.int16), ref.view(torch.int16))


def test_noalloc_rejects_shapes_beyond_the_scratch():
    # 2 * 576 * (32768 + 32768) bytes > 48 MiB: refused before anything is read or launched.
    fake = ctypes.c_void_p(0x7F0000000000)
    st = lg.lib.lg_lora_linear_noalloc(fake, fake, fake, fake, ctypes.c_void_p(0x7F1000000000), 128, 32768,
                                       32768, 576, None)
    assert st == lg.LG_ERR_WORKSPACE


_CONTEXT_SCRIPT = r"""
import ctypes, sys
import numpy as np
sys.path.insert(0, sys.argv[1])
import lora_gemm_b200 as lg

cu = ctypes.CDLL("libcuda.so.1")


def ck(r, what):
    assert r == 0, f"{what}: CUresult {r}"


ck(cu.cuInit(0), "cuInit")
dev = ctypes.c_int()
ck(cu.cuDeviceGet(ctypes.byref(dev), 0), "cuDeviceGet")
M, K, N, R = 200, 512, 320, 576
rng = np.random.default_rng(0)
f32_to_bf16 = lambda a: (a.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
host = {
    "x": f32_to_bf16(rng.standard_normal((M, K))),
    "W": f32_to_bf16(rng.standard_normal((N, K)) * K ** -0.5),
    "A": (rng.standard_normal((R, K)) * K ** -0.5).astype(np.float32),
    "B": (rng.standard_normal((N, R)) * 0.1).astype(np.float32),
}
ws_bytes = lg.lora_linear_workspace_size(M, K, N, R)


def run_in_current_context():
    bufs = {}
    for name, a in host.items():
        p = ctypes.c_uint64()
        ck(cu.cuMemAlloc_v2(ctypes.byref(p), ctypes.c_size_t(a.nbytes)), "cuMemAlloc")
        ck(cu.cuMemcpyHtoD_v2(p, a.ctypes.data_as(ctypes.c_void_p), ctypes.c_size_t(a.nbytes)), "HtoD")
        bufs[name] = p
    for name, nbytes in (("y0", 2 * M * N), ("y1", 2 * M * N), ("ws", ws_bytes)):
        p = ctypes.c_uint64()
        ck(cu.cuMemAlloc_v2(ctypes.byref(p), ctypes.c_size_t(nbytes)), "cuMemAlloc")
        bufs[name] = p
    P = lambda n: ctypes.c_void_p(bufs[n].value)
    st = lg.lib.lg_lora_linear_noalloc(P("x"), P("W"), P("A"), P("B"), P("y0"), M, K, N, R, None)
    assert st == 0, lg.status_string(st)
    st = lg.lib.lg_lora_linear(P("x"), P("W"), P("A"), P("B"), P("y1"), M, K, N, R, P("ws"), ws_bytes, None)
    assert st == 0, lg.status_string(st)
    assert lg.lib.lg_get_last_device_error(None) == 0
    out = []
    for n in ("y0", "y1"):
        h = np.empty((M, N), np.uint16)
        ck(cu.cuMemcpyDtoH_v2(h.ctypes.data_as(ctypes.c_void_p), bufs[n], ctypes.c_size_t(h.nbytes)), "DtoH")
        out.append(h)
    for p in bufs.values():
        ck(cu.cuMemFree_v2(p), "cuMemFree")
    assert np.array_equal(out[0], out[1]), "noalloc differs from lg_lora_linear"
    return out[0]


primary = ctypes.c_void_p()
ck(cu.cuDevicePrimaryCtxRetain(ctypes.byref(primary), dev), "retain")
ck(cu.cuCtxSetCurrent(primary), "set primary")
y_primary = run_in_current_context()
second = ctypes.c_void_p()
ck(cu.cuCtxCreate_v2(ctypes.byref(second), 0, dev), "create")
y_second = run_in_current_context()
ck(cu.cuCtxDestroy_v2(second), "destroy")
ck(cu.cuCtxSetCurrent(primary), "set primary again")
y_again = run_in_current_context()
assert np.array_equal(y_primary, y_second) and np.array_equal(y_primary, y_again)
print("CONTEXTS OK")
"""


def test_noalloc_follows_the_current_context():
    """The cached scratch address belongs to the context it was looked up
    in: under a second context (created with the driver API, as a plugin
    host may do) the call looks it up again, and back under the primary
    context too.  Runs in a child process without torch's CUDA state."""
    out = subprocess.run([sys.executable, "-c", _CONTEXT_SCRIPT, ROOT], capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0 and "CONTEXTS OK" in out.stdout, out.stdout[-2000:] + out.stderr[-3000:]
