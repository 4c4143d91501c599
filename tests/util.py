"""Comparison helpers for the parity tests (no method arithmetic here)."""

import numpy as np


def f32_ordered(a):
    """Map FP32 values to integers whose difference counts ulps (+0 and -0 coincide)."""
    i = np.asarray(a, dtype=np.float32).view(np.int32).astype(np.int64)
    return np.where(i < 0, -(i & 0x7FFFFFFF), i)


def ulp_diff(a, b):
    """Number of FP32 steps between a and b, element by element."""
    return np.abs(f32_ordered(a) - f32_ordered(b))


def ulp_of(x):
    """Size of one FP32 ulp at |x| (the gap to the next float away from zero)."""
    x = np.abs(np.asarray(x, dtype=np.float32))
    return (np.nextafter(x, np.float32(np.inf)) - x).astype(np.float64)


def rel_fro(a, b):
    """||a - b||_F / ||b||_F in FP64."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))
