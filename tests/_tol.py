"""Tolerance helpers shared by the tests (no method arithmetic)."""
import numpy as np


def ulp_bf16(x):
    """Spacing of bf16 numbers at |x|: 2^(floor(log2|x|) - 7), floored at the
    smallest normal spacing."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    a = np.maximum(a, 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


def bf16_bits_to_f64(h):
    h = np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16
    return h.view(np.float32).astype(np.float64)
