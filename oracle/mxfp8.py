"""MXFP8 (E4M3 elements, E8M0 block scales) and the MXFP8 merged-LoRA linear layer
(oracle side, FP64).  TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: "Open-H3-Regenerate-2K: High-Resolution Video Refinement with Few-Step
Diffusion" (agientry.com), section "Where the 3.9x speedup comes from": the
optimized engine runs the transformer's linear layers as MXFP8 GEMMs, with the
activations re-quantized at every stage.  The pages give no format details;
this module takes the published Open Compute Project "Microscaling (MX)
Formats" definition (v1.0) as the plainest reading of "MXFP8":

* a block is 32 consecutive values along the reduction axis K;
* the block scale is X = 2^e with e = floor(log2(max |V_i|)) - 8 (8 being the
  exponent of the largest normal E4M3 number, 448 = 1.75 * 2^8), clamped to
  the E8M0 range [-127, 127] and stored as the byte e + 127; an all-zero block
  gets e = -127 (this reading: the spec leaves log2(0) open);
* each element is V_i / X converted to E4M3 (OCP 8-bit float "E4M3FN": bias 7,
  3 mantissa bits, no infinities, largest finite 448, the all-ones code NaN)
  by round-to-nearest-even, magnitudes beyond 448 saturating to +-448 (the
  spec leaves overflow to the implementation; this reading saturates).

The MXFP8 layer keeps the LoRA path of ``oracle.lora.lora_linear`` unchanged
(bf16 activations, the merged factors) and replaces only the base term:

    y = deq(x) deq(W)^T + (x A_cat^T) B_cat^T

with deq(.) the exact value of the quantized operand (code value times 2^e).
"""

import math

import numpy as np

E4M3_MAX = 448.0
E8M0_MIN_EXP = -127
E8M0_MAX_EXP = 127
BLOCK = 32


def e4m3_decode(code):
    """Value of one E4M3 code (0..255) as a Python float; NaN for the two NaN codes."""
    code = int(code)
    sign = -1.0 if code & 0x80 else 1.0
    exp = (code >> 3) & 0xF
    man = code & 0x7
    if exp == 0xF and man == 0x7:
        return math.nan
    if exp == 0:
        return sign * (man / 8.0) * 2.0 ** -6
    return sign * (1.0 + man / 8.0) * 2.0 ** (exp - 7)


# Non-negative finite codes and their values, ascending (code 0x00..0x7E).
_POS_CODES = np.arange(0x7F, dtype=np.int64)
_POS_VALUES = np.array([e4m3_decode(c) for c in _POS_CODES], dtype=np.float64)


def e4m3_encode(v):
    """Nearest E4M3 code to the float v (round to nearest, ties to the even
    code, i.e. the even mantissa), saturating beyond 448; the sign of zero is
    kept.  Plain search over the 127 non-negative finite codes."""
    v = float(v)
    if math.isnan(v):
        raise ValueError("NaN has no MXFP8 encoding here")
    sign = 0x80 if math.copysign(1.0, v) < 0 else 0
    a = abs(v)
    if a >= E4M3_MAX:
        return sign | 0x7E
    d = np.abs(_POS_VALUES - a)
    best = np.flatnonzero(d == d.min())
    if best.size == 1:
        code = int(best[0])
    else:  # exactly halfway between two neighbours: the even code
        code = int(best[0]) if best[0] % 2 == 0 else int(best[1])
    return sign | code


def block_exponent(block):
    """Shared exponent e of one block of values (floats): floor(log2 amax) - 8,
    clamped to [-127, 127]; -127 for an all-zero block."""
    amax = max(abs(float(v)) for v in block)
    if amax == 0.0:
        return E8M0_MIN_EXP
    m, ex = math.frexp(amax)  # amax = m 2^ex, m in [0.5, 1): floor(log2 amax) = ex - 1
    e = (ex - 1) - 8
    return min(max(e, E8M0_MIN_EXP), E8M0_MAX_EXP)


def e4m3_encode_array(a):
    """Vectorised e4m3_encode over an FP64 array (same rule: nearest code,
    ties to the even code, saturation at 448, sign of zero kept): the two
    neighbours come from a sorted search of the value table."""
    a = np.asarray(a, dtype=np.float64)
    if np.isnan(a).any():
        raise ValueError("NaN has no MXFP8 encoding here")
    sign = np.where(np.signbit(a), 0x80, 0).astype(np.int64)
    m = np.abs(a)
    hi = np.clip(np.searchsorted(_POS_VALUES, m, side="left"), 0, len(_POS_VALUES) - 1)
    lo = np.clip(hi - 1, 0, len(_POS_VALUES) - 1)
    d_hi = np.abs(_POS_VALUES[hi] - m)
    d_lo = np.abs(m - _POS_VALUES[lo])
    code = np.where(d_lo < d_hi, lo, hi)
    tie = (d_lo == d_hi) & (lo != hi)
    code = np.where(tie, np.where(lo % 2 == 0, lo, hi), code)
    code = np.where(m >= E4M3_MAX, 0x7E, code)
    return (sign | code).astype(np.uint8)


def block_exponents(V):
    """block_exponent of every 32-block of the rows of V [rows, K]."""
    V = np.asarray(V, dtype=np.float64)
    rows, K = V.shape
    amax = np.abs(V).reshape(rows, K // BLOCK, BLOCK).max(axis=2)
    _, ex = np.frexp(amax)
    e = np.clip(ex.astype(np.int64) - 1 - 8, E8M0_MIN_EXP, E8M0_MAX_EXP)
    return np.where(amax == 0.0, E8M0_MIN_EXP, e).astype(np.int32)


def mx_quantize(V):
    """Quantize the rows of V [rows, K] (K a multiple of 32) along K.

    Returns (codes uint8 [rows, K], exps int32 [rows, K / 32]); the E8M0 scale
    byte of a block is exps + 127."""
    V = np.asarray(V, dtype=np.float64)
    rows, K = V.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 32")
    exps = block_exponents(V)
    scaled = np.ldexp(V, -np.repeat(exps, BLOCK, axis=1).astype(np.int64))
    return e4m3_encode_array(scaled), exps


def mx_quantize_scalar(V):
    """mx_quantize element by element with the scalar rules (the slow form the
    vectorised one is pinned against)."""
    V = np.asarray(V, dtype=np.float64)
    rows, K = V.shape
    codes = np.zeros((rows, K), dtype=np.uint8)
    exps = np.zeros((rows, K // BLOCK), dtype=np.int32)
    for r in range(rows):
        for b in range(K // BLOCK):
            blk = V[r, BLOCK * b:BLOCK * (b + 1)]
            e = block_exponent(blk)
            exps[r, b] = e
            for i, v in enumerate(blk):
                codes[r, BLOCK * b + i] = e4m3_encode(math.ldexp(float(v), -e))
    return codes, exps


def mx_dequantize(codes, exps):
    """Exact values of quantized rows: code value times 2^e of its block (FP64)."""
    codes = np.asarray(codes)
    exps = np.asarray(exps)
    vals = _DECODE_ALL[codes.astype(np.int64)]
    scale = np.ldexp(1.0, np.repeat(exps, BLOCK, axis=1).astype(np.int64))
    return vals * scale


_DECODE_ALL = np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)


def lora_linear_mxfp8(x, W, A_cat, B_cat):
    """y = deq(Q(x)) deq(Q(W))^T + (x A_cat^T) B_cat^T in FP64, x and W
    quantized along K as above, the LoRA term from the unquantized x."""
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    xq = mx_dequantize(*mx_quantize(x))
    wq = mx_dequantize(*mx_quantize(W))
    y = xq @ wq.T
    if A_cat is not None and np.asarray(A_cat).shape[0] > 0:
        A = np.asarray(A_cat, dtype=np.float64)
        B = np.asarray(B_cat, dtype=np.float64)
        y = y + (x @ A.T) @ B.T
    return y


def silu(g):
    """SiLU, g * sigmoid(g) = g / (1 + e^-g), in FP64 (e^-g overflows to inf for
    g < -709, giving the limit 0 correctly)."""
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def swiglu_mxfp8(x, W2, A_cat, B_cat):
    """The MLP input projection with SwiGLU and the activation quantizer fused
    ("Open-H3-Regenerate-2K: High-Resolution Video Refinement with Few-Step
    Diffusion", section "Where the 3.9x speedup comes from": fused SwiGLU with
    MXFP8, one-pass activation quantization).  W2 [2F, K] holds the gate rows
    followed by the up rows (this library's reading: the pages only note that
    the gate/up layout differs between formats); B_cat [2F, R] likewise.

        z = lora_linear_mxfp8(x, W2, A_cat, B_cat)      [M, 2F]
        s = silu(z[:, :F]) * z[:, F:]                   [M, F]

    Returns (s in FP64, mx_quantize(s))."""
    z = lora_linear_mxfp8(x, W2, A_cat, B_cat)
    F = z.shape[1] // 2
    s = silu(z[:, :F]) * z[:, F:]
    return s, mx_quantize(s)
