"""Pins of the MXFP8 oracle (oracle/mxfp8.py) against facts fixed outside it:
the E4M3 bit layout of the OCP 8-bit float format, PyTorch's independent
float8_e4m3fn conversion (round to nearest even) for in-range values, the
round-to-nearest-even rule at exact midpoints, saturation, the block-exponent
definition, the quantization error bound of a 3-bit mantissa and brute-force
loops on tiny layers."""

import math

import numpy as np
import pytest
import torch

from oracle import lora as olora
from oracle import mxfp8 as mx

FINITE = [c for c in range(256) if c not in (0x7F, 0xFF)]


def test_decode_known_codes():
    assert mx.e4m3_decode(0x00) == 0.0
    assert math.copysign(1.0, mx.e4m3_decode(0x80)) == -1.0
    assert mx.e4m3_decode(0x01) == 2.0 ** -9          # smallest subnormal
    assert mx.e4m3_decode(0x07) == 7 * 2.0 ** -9      # largest subnormal
    assert mx.e4m3_decode(0x08) == 2.0 ** -6          # smallest normal
    assert mx.e4m3_decode(0x38) == 1.0
    assert mx.e4m3_decode(0x39) == 1.125
    assert mx.e4m3_decode(0x7E) == 448.0              # largest finite
    assert mx.e4m3_decode(0xFE) == -448.0
    assert math.isnan(mx.e4m3_decode(0x7F)) and math.isnan(mx.e4m3_decode(0xFF))


def test_decode_matches_torch_float8_e4m3fn():
    codes = torch.tensor(FINITE, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = np.array([mx.e4m3_decode(c) for c in FINITE])
    assert np.array_equal(ref, ours)


def test_encode_inverts_decode():
    for c in FINITE:
        assert mx.e4m3_encode(mx.e4m3_decode(c)) == c, hex(c)


def test_midpoints_round_to_even():
    vals = [mx.e4m3_decode(c) for c in range(0x7F)]
    for c in range(0x7E):
        mid = 0.5 * (vals[c] + vals[c + 1])
        even = c if c % 2 == 0 else c + 1
        assert mx.e4m3_encode(mid) == even, (c, mid)
        assert mx.e4m3_encode(-mid) == 0x80 | even
        assert mx.e4m3_encode(math.nextafter(mid, 0.0)) == c
        assert mx.e4m3_encode(math.nextafter(mid, math.inf)) == c + 1


def test_saturation():
    for v in (448.0, 449.0, 463.9, 464.0, 480.0, 1e6, 3.0e38):
        assert mx.e4m3_encode(v) == 0x7E
        assert mx.e4m3_encode(-v) == 0xFE


def test_encode_matches_torch_in_range():
    rng = np.random.default_rng(7)
    mags = np.ldexp(rng.uniform(1.0, 2.0, 20000), rng.integers(-12, 9, 20000)).astype(np.float32)
    v = (mags * rng.choice([-1.0, 1.0], 20000)).astype(np.float32)
    v = v[np.abs(v) < 448.0]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = mx.e4m3_encode_array(v.astype(np.float64))
    assert np.array_equal(ref, ours)
    scalar = np.array([mx.e4m3_encode(float(t)) for t in v[:3000]], dtype=np.uint8)
    assert np.array_equal(scalar, ours[:3000])


def test_block_exponent_definition():
    assert mx.block_exponent([1.0] + [0.0] * 31) == -8
    assert mx.block_exponent([0.0] * 32) == -127
    assert mx.block_exponent([-448.0]) == 0
    assert mx.block_exponent([511.9]) == 0
    assert mx.block_exponent([512.0]) == 1
    assert mx.block_exponent([2.0 ** -130]) == -127       # clamped to the E8M0 range
    assert mx.block_exponent([2.0 ** 140]) == 127


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_vectorised_quantizer_equals_scalar(seed):
    rng = np.random.default_rng(seed)
    V = rng.standard_normal((6, 128)) * np.ldexp(1.0, rng.integers(-30, 30, (6, 1)))
    V[0, :32] = 0.0                        # an all-zero block
    V[1, 32:64] = rng.choice([-1.0, 1.0], 32) * 2.0 ** -140
    V[2, 64] = 480.0 * 2.0 ** -2           # saturates after scaling
    a = mx.mx_quantize(V)
    b = mx.mx_quantize_scalar(V)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_scaled_block_maximum_and_error_bound():
    rng = np.random.default_rng(3)
    V = rng.standard_normal((64, 256)) * np.ldexp(1.0, rng.integers(-10, 10, (64, 1)))
    codes, exps = mx.mx_quantize(V)
    D = mx.mx_dequantize(codes, exps)
    amax = np.abs(V).reshape(64, 8, 32).max(axis=2)
    scaled = amax / np.ldexp(1.0, exps)
    assert ((scaled >= 256.0) & (scaled < 512.0)).all()
    scale = np.ldexp(1.0, np.repeat(exps, 32, axis=1))
    normal = (np.abs(V) / scale >= 2.0 ** -6) & (np.abs(V) / scale <= 448.0)
    assert (np.abs(D - V)[normal] <= 2.0 ** -4 * np.abs(V)[normal]).all()
    sub = np.abs(V) / scale < 2.0 ** -6
    assert (np.abs(D - V)[sub] <= 2.0 ** -10 * scale[sub]).all()
    sat = np.abs(V) / scale > 448.0
    assert np.array_equal(np.abs(D[sat]), 448.0 * scale[sat])


def test_linear_brute_force_tiny():
    rng = np.random.default_rng(11)
    M, K, N, R = 3, 64, 5, 4
    x = rng.standard_normal((M, K))
    W = rng.standard_normal((N, K)) * 0.1
    A = rng.standard_normal((R, K)) * 0.1
    B = rng.standard_normal((N, R)) * 0.1
    cx, ex = mx.mx_quantize_scalar(x)
    cw, ew = mx.mx_quantize_scalar(W)
    y = mx.lora_linear_mxfp8(x, W, A, B)
    for m in range(M):
        for n in range(N):
            base = 0.0
            for k in range(K):
                base += (mx.e4m3_decode(cx[m, k]) * 2.0 ** ex[m, k // 32]) * (
                    mx.e4m3_decode(cw[n, k]) * 2.0 ** ew[n, k // 32])
            lora = 0.0
            for r in range(R):
                h = sum(x[m, k] * A[r, k] for k in range(K))
                lora += h * B[n, r]
            assert abs(y[m, n] - (base + lora)) <= 1e-12 * (1.0 + abs(base) + abs(lora))


def test_linear_close_to_unquantized_and_rank_zero():
    rng = np.random.default_rng(12)
    M, K, N, R = 64, 256, 96, 32
    x = rng.standard_normal((M, K))
    W = rng.standard_normal((N, K)) / np.sqrt(K)
    A = rng.standard_normal((R, K)) / np.sqrt(K)
    B = rng.standard_normal((N, R)) * 0.1
    y = mx.lora_linear_mxfp8(x, W, A, B)
    ref = olora.lora_linear(x, W, A, B)
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert 1e-3 < rel < 5e-2
    y0 = mx.lora_linear_mxfp8(x, W, np.zeros((0, K)), np.zeros((N, 0)))
    assert np.allclose(y0, mx.mx_dequantize(*mx.mx_quantize(x)) @ mx.mx_dequantize(*mx.mx_quantize(W)).T, rtol=0,
                       atol=1e-12)


def test_silu_against_torch_and_limits():
    g = np.concatenate([np.linspace(-30, 30, 2001), [0.0, 800.0, -800.0, 1e-300]])
    ours = mx.silu(g)
    ref = torch.nn.functional.silu(torch.from_numpy(g)).numpy()
    assert np.allclose(ours, ref, rtol=1e-14, atol=1e-300)
    assert mx.silu(0.0) == 0.0
    assert mx.silu(800.0) == 800.0
    assert mx.silu(-800.0) == 0.0


def test_swiglu_brute_force_tiny():
    rng = np.random.default_rng(21)
    M, K, F, R = 3, 64, 32, 4
    x = rng.standard_normal((M, K))
    W2 = rng.standard_normal((2 * F, K)) * 0.2
    A = rng.standard_normal((R, K)) * 0.1
    B = rng.standard_normal((2 * F, R)) * 0.1
    s, (codes, exps) = mx.swiglu_mxfp8(x, W2, A, B)
    z = mx.lora_linear_mxfp8(x, W2, A, B)
    for m in range(M):
        for j in range(F):
            g, u = z[m, j], z[m, F + j]
            assert abs(s[m, j] - g / (1.0 + math.exp(-g)) * u) <= 1e-14 * (1 + abs(s[m, j]))
    c2, e2 = mx.mx_quantize_scalar(s)
    assert np.array_equal(codes, c2) and np.array_equal(exps, e2)
