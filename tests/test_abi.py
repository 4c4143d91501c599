"""The C ABI library loads, exports every declared symbol, and validates
arguments on the host before touching a GPU (these tests need no GPU: every
call here fails validation, so nothing is launched)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lora_gemm.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lg_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for must in ("lg_lora_merge", "lg_lora_linear", "lg_renoise", "lg_euler_step"):
        assert must in names


def test_library_exports_every_declared_symbol():
    import lora_gemm_b200 as lg

    lib = ctypes.CDLL(lg.LIB_PATH)
    for name in _declared_functions():
        assert hasattr(lib, name), name
    assert sorted(lg.EXPORTED_SYMBOLS) == _declared_functions()


def test_status_strings_and_version():
    import lora_gemm_b200 as lg

    for s in range(8):
        assert lg.status_string(s) and lg.status_string(s) != "unknown status"
    assert lg.status_string(99) == "unknown status"
    assert lg.version() >= 10000


def test_workspace_size_host_arithmetic():
    import lora_gemm_b200 as lg

    def a256(v):
        return (v + 255) // 256 * 256

    assert lg.lora_linear_workspace_size(532800, 7168, 7168, 576) == a256(2 * 576 * 7168) * 2
    assert lg.lora_linear_workspace_size(10, 7168, 21504, 576) == a256(2 * 576 * 7168) + a256(2 * 21504 * 576)
    assert lg.lora_linear_workspace_size(10, 1024, 1024, 0) == 0
    for bad in [(10, 100, 64, 64), (10, 64, 100, 64), (10, 64, 16, 64), (10, 64, 64, 32), (10, 64, 64, 640),
                (-1, 64, 64, 64)]:
        assert lg.lora_linear_workspace_size(*bad) == 0


P = ctypes.c_void_p
A16 = P(0x7F0000000000)  # fake, 16-byte aligned, never dereferenced
A16b = P(0x7F0000100000)
MIS = P(0x7F0000000004)


def test_host_validation_elementwise():
    import lora_gemm_b200 as lg

    L = lg.lib
    assert L.lg_renoise(None, None, 16, 0.5, 0, 0, None) == lg.LG_ERR_INVALID_ARG
    assert L.lg_renoise(A16, A16b, 16, 1.5, 0, 0, None) == lg.LG_ERR_INVALID_ARG
    assert L.lg_renoise(A16, A16b, 16, -0.1, 0, 0, None) == lg.LG_ERR_INVALID_ARG
    assert L.lg_renoise(A16, A16b, 16, float("nan"), 0, 0, None) == lg.LG_ERR_INVALID_ARG
    assert L.lg_renoise(A16, A16b, 16, 0.5, 0, 2, None) == lg.LG_ERR_INVALID_ARG
    assert L.lg_renoise(MIS, A16b, 16, 0.5, 0, 0, None) == lg.LG_ERR_MISALIGNED
    assert L.lg_renoise(A16, P(A16.value + 16), 16, 0.5, 0, 0, None) == lg.LG_ERR_INVALID_ARG  # partial overlap
    assert L.lg_renoise(None, None, 0, 0.5, 0, 0, None) == lg.LG_OK  # empty: nothing to do
    assert L.lg_euler_step(None, A16b, 16, 0.9, 0.8, None) == lg.LG_ERR_INVALID_ARG
    assert L.lg_euler_step(A16, A16, 16, 0.9, 0.8, None) == lg.LG_ERR_INVALID_ARG  # x and v overlap
    assert L.lg_euler_step(A16, MIS, 16, 0.9, 0.8, None) == lg.LG_ERR_MISALIGNED
    assert L.lg_euler_step(A16, A16b, 16, float("inf"), 0.8, None) == lg.LG_ERR_INVALID_ARG
    assert L.lg_euler_step(None, None, 0, 0.9, 0.8, None) == lg.LG_OK
    assert L.lg_philox_u32(None, 4, 0, 0, None) == lg.LG_ERR_INVALID_ARG
    assert L.lg_philox_u32(MIS, 4, 0, 0, None) == lg.LG_ERR_MISALIGNED
    assert L.lg_philox_u32(A16, -1, 0, 0, None) == lg.LG_ERR_INVALID_ARG
    assert L.lg_philox_normal(A16, 8, 0, 3, None) == lg.LG_ERR_INVALID_ARG
    assert L.lg_philox_normal(None, 0, 0, 0, None) == lg.LG_OK


def test_host_validation_lora_linear():
    import lora_gemm_b200 as lg

    L = lg.lib
    ws = P(0x7F0040000000)
    y = P(0x7F0080000000)
    big = 1 << 30

    def call(x=A16, W=A16b, A=P(0x7F0010000000), B=P(0x7F0020000000), y=y, M=256, K=128, N=128, R=64, ws=ws,
             ws_bytes=big):
        return L.lg_lora_linear(x, W, A, B, y, M, K, N, R, ws, ws_bytes, None)

    assert call(K=100) == lg.LG_ERR_UNSUPPORTED_SHAPE
    assert call(N=80) == lg.LG_ERR_UNSUPPORTED_SHAPE
    assert call(N=16) == lg.LG_ERR_UNSUPPORTED_SHAPE
    assert call(R=32) == lg.LG_ERR_UNSUPPORTED_SHAPE
    assert call(R=640) == lg.LG_ERR_UNSUPPORTED_SHAPE
    assert call(M=1 << 31) == lg.LG_ERR_UNSUPPORTED_SHAPE
    assert call(M=-1) == lg.LG_ERR_INVALID_ARG
    assert call(x=None) == lg.LG_ERR_INVALID_ARG
    assert call(A=None) == lg.LG_ERR_INVALID_ARG
    assert call(x=MIS) == lg.LG_ERR_MISALIGNED
    assert call(ws=None) == lg.LG_ERR_WORKSPACE
    assert call(ws_bytes=16) == lg.LG_ERR_WORKSPACE
    assert call(y=P(A16.value + 64)) == lg.LG_ERR_INVALID_ARG  # y overlaps x
    assert call(M=0) == lg.LG_OK  # empty: nothing to do
    assert call(A=None, B=None, R=0, ws=None, ws_bytes=0, M=0) == lg.LG_OK


def test_host_validation_merge():
    import lora_gemm_b200 as lg

    L = lg.lib
    ptrs = (P * 3)(0x7F0000000000, 0x7F0001000000, 0x7F0002000000)
    bptrs = (P * 3)(0x7F0003000000, 0x7F0004000000, 0x7F0005000000)
    ranks = (ctypes.c_int * 3)(384, 128, 64)
    bad_ranks = (ctypes.c_int * 3)(384, 126, 64)
    scales = (ctypes.c_float * 3)(1.0, 1.0, 1.0)
    Ac, Bc = P(0x7F0010000000), P(0x7F0020000000)
    assert L.lg_lora_merge(0, ptrs, bptrs, ranks, scales, 64, 64, Ac, Bc, None) == lg.LG_ERR_INVALID_ARG
    assert L.lg_lora_merge(9, ptrs, bptrs, ranks, scales, 64, 64, Ac, Bc, None) == lg.LG_ERR_INVALID_ARG
    assert L.lg_lora_merge(3, ptrs, bptrs, bad_ranks, scales, 64, 64, Ac, Bc, None) == lg.LG_ERR_UNSUPPORTED_SHAPE
    assert L.lg_lora_merge(3, ptrs, bptrs, ranks, scales, 66, 64, Ac, Bc, None) == lg.LG_ERR_UNSUPPORTED_SHAPE
    assert L.lg_lora_merge(3, ptrs, bptrs, ranks, scales, 64, 64, MIS, Bc, None) == lg.LG_ERR_MISALIGNED
    assert L.lg_lora_merge(3, ptrs, bptrs, ranks, scales, 64, 64, None, Bc, None) == lg.LG_ERR_INVALID_ARG


def test_host_validation_fused_and_mxfp8_entry_points():
    """Argument checks of the MXFP8, SwiGLU and Euler entry points run before
    anything touches a device (fake pointers, no GPU needed)."""
    import lora_gemm_b200 as lg

    L = lg.lib
    ws, out, sc = P(0x7F0040000000), P(0x7F0080000000), P(0x7F00C0000000)
    xq, xs, wq, wsf = P(0x7F0100000000), P(0x7F0140000000), P(0x7F0180000000), P(0x7F01C0000000)
    A, B = P(0x7F0010000000), P(0x7F0020000000)
    big = 1 << 30

    def mx(M=256, K=128, N=128, R=64, x=A16, y=out, ws_bytes=big, xq=xq):
        return L.lg_lora_linear_mxfp8(x, xq, xs, wq, wsf, A, B, y, M, K, N, R, ws, ws_bytes, None)

    assert mx(K=192) == lg.LG_ERR_UNSUPPORTED_SHAPE          # K not a multiple of 128
    assert mx(N=48) == lg.LG_ERR_UNSUPPORTED_SHAPE
    assert mx(xq=None) == lg.LG_ERR_INVALID_ARG
    assert mx(xq=MIS) == lg.LG_ERR_MISALIGNED
    assert mx(y=P(xq.value + 1024)) == lg.LG_ERR_INVALID_ARG  # y overlaps the x codes
    assert mx(ws_bytes=0) == lg.LG_ERR_WORKSPACE
    assert mx(M=0) == lg.LG_OK

    def sw(M=256, K=128, F=128, R=64, codes=out, scales=sc):
        return L.lg_lora_linear_swiglu_mxfp8(A16, xq, xs, wq, wsf, A, B, codes, scales, M, K, F, R, ws, big, None)

    assert sw(F=96) == lg.LG_ERR_UNSUPPORTED_SHAPE           # F not a multiple of 128
    assert sw(codes=None) == lg.LG_ERR_INVALID_ARG
    assert sw(scales=MIS) == lg.LG_ERR_MISALIGNED
    assert sw(scales=P(out.value + 64)) == lg.LG_ERR_INVALID_ARG  # scales overlap the codes
    assert sw(M=0) == lg.LG_OK

    def eu(M=256, K=128, N=24, R=64, z=out, zb=sc, T=128, s0=0.857, s1=0.667, ws_bytes=big):
        return L.lg_lora_linear_euler(A16, A16b, A, B, z, zb, M, K, N, R, T, s0, s1, ws, ws_bytes, None)

    assert eu(N=0) == lg.LG_ERR_UNSUPPORTED_SHAPE
    assert eu(K=96) == lg.LG_ERR_UNSUPPORTED_SHAPE
    assert eu(T=100) == lg.LG_ERR_INVALID_ARG                 # M not a multiple of the frame
    assert eu(T=0) == lg.LG_ERR_INVALID_ARG
    assert eu(s1=float("nan")) == lg.LG_ERR_INVALID_ARG
    assert eu(z=None) == lg.LG_ERR_INVALID_ARG
    assert eu(z=MIS) == lg.LG_ERR_MISALIGNED
    assert eu(zb=P(out.value + 256)) == lg.LG_ERR_INVALID_ARG  # bf16 copy overlaps z
    assert eu(z=P(A16.value + 256)) == lg.LG_ERR_INVALID_ARG   # z overlaps x
    assert eu(ws_bytes=16) == lg.LG_ERR_WORKSPACE
    assert eu(M=0) == lg.LG_OK
    assert eu(M=0, zb=None) == lg.LG_OK

    def a256(v):
        return (v + 255) // 256 * 256

    assert lg.lora_linear_euler_workspace_size(532800, 7168, 24, 576) == a256(2 * 576 * 7168) + a256(2 * 24 * 576)
    assert lg.lora_linear_euler_workspace_size(10, 7168, 24, 0) == 0
    assert lg.lora_linear_euler_workspace_size(10, 100, 24, 64) == 0
    assert L.lg_mx_quantize(None, 4, 128, out, sc, None) == lg.LG_ERR_INVALID_ARG
    assert L.lg_mx_quantize(A16, 4, 96, out, sc, None) == lg.LG_ERR_UNSUPPORTED_SHAPE


def test_mx_scale_bytes_host_arithmetic():
    """One E8M0 byte per 32 values along K, rows padded to the 128-row groups
    of the blocked layout (the layout the block-scaled MMAs read)."""
    import lora_gemm_b200 as lg

    assert lg.mx_scale_bytes(128, 128) == 128 * 4
    assert lg.mx_scale_bytes(1, 128) == 128 * 4
    assert lg.mx_scale_bytes(129, 256) == 256 * 8
    assert lg.mx_scale_bytes(532800, 7168) == (532800 + 127) // 128 * 128 * 224
    assert lg.mx_scale_bytes(0, 128) == 0
    for bad in [(10, 96), (10, 64), (-1, 128), (10, 0)]:
        assert lg.mx_scale_bytes(*bad) == 0


def test_noalloc_reports_the_same_status_as_lg_lora_linear():
    """lg_lora_linear_noalloc runs lg_lora_linear's argument checks before its
    own scratch limit and before any CUDA call, so a bad argument gives the
    same status from both entry points (CPU: nothing here reaches a device)."""
    import ctypes

    import lora_gemm_b200 as lg

    L = lg.lib
    base = 0x7F0000000000
    x, W, A, B, y, ws = (ctypes.c_void_p(base + i * (1 << 36)) for i in range(6))
    ws_bytes = 1 << 30
    cases = {
        "null x": ((None, W, A, B, y, 256, 1024, 1024, 576), lg.LG_ERR_INVALID_ARG),
        "null y": ((x, W, A, B, None, 256, 1024, 1024, 576), lg.LG_ERR_INVALID_ARG),
        "null A_cat": ((x, W, None, B, y, 256, 1024, 1024, 576), lg.LG_ERR_INVALID_ARG),
        "misaligned x": ((ctypes.c_void_p(base + 8), W, A, B, y, 256, 1024, 1024, 576), lg.LG_ERR_MISALIGNED),
        "K not a multiple of 64": ((x, W, A, B, y, 256, 1000, 1024, 576), lg.LG_ERR_UNSUPPORTED_SHAPE),
        "rank not a multiple of 64": ((x, W, A, B, y, 256, 1024, 1024, 96), lg.LG_ERR_UNSUPPORTED_SHAPE),
        "y overlaps x": ((x, W, A, B, ctypes.c_void_p(base + 1024), 256, 1024, 1024, 576), lg.LG_ERR_INVALID_ARG),
        "negative M": ((x, W, A, B, y, -1, 1024, 1024, 576), lg.LG_ERR_INVALID_ARG),
    }
    for name, (args, want) in cases.items():
        a = args[:9]
        got_ws = L.lg_lora_linear(*a, ws, ws_bytes, None)
        got_na = L.lg_lora_linear_noalloc(*a, None)
        assert got_ws == got_na == want, f"{name}: lg_lora_linear {got_ws}, noalloc {got_na}, want {want}"
    # An empty batch with a valid shape launches nothing and needs no device.
    assert L.lg_lora_linear_noalloc(x, W, A, B, y, 0, 1024, 1024, 576, None) == lg.LG_OK
    # Valid arguments but a shape beyond the built-in scratch: refused as a too-small workspace would be.
    assert L.lg_lora_linear_noalloc(x, W, A, B, y, 0, 32768, 32768, 576, None) == lg.LG_ERR_WORKSPACE
    assert L.lg_lora_linear(x, W, A, B, y, 0, 32768, 32768, 576, ws, lg.LG_NOALLOC_SCRATCH_BYTES, None) == \
        lg.LG_ERR_WORKSPACE



def test_tuning_knobs_validate_their_range():
    import lora_gemm_b200 as lg

    L = lg.lib
    for v in (3, 16, -1):
        assert L.lg_set_cluster_size(v) == lg.LG_ERR_INVALID_ARG
    for v in (-1, 3):
        assert L.lg_set_kernel_variant(v) == lg.LG_ERR_INVALID_ARG
