"""Exact bf16 <-> float64 helpers for the oracle (test infrastructure only).

A bf16 value is the upper 16 bits of an IEEE-754 binary32 value, so widening
is exact: put the 16 bits in the top half of a 32-bit word, read it as
float32, then convert to float64 (also exact).  The oracle keeps the KV pool
as raw uint16 bit patterns so that copies are checked byte for byte and NaN
payloads or negative zero survive.
"""

import numpy as np

BF16_QNAN = np.uint16(0x7FC0)


def as_u16(a):
    """View an integer array of bf16 bit patterns as uint16 (no copy if possible)."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return a
    if a.dtype == np.int16:
        return a.view(np.uint16)
    raise TypeError(f"expected uint16/int16 bf16 bit patterns, got {a.dtype}")


def to_f64(bits):
    """Widen bf16 bit patterns (uint16/int16 array) exactly to float64."""
    u = as_u16(bits).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def from_f64_exact(x):
    """Encode float64 values that are exactly representable in bf16.

    Raises if any value would need rounding: the oracle never rounds inputs,
    it only encodes hand-written exact test values.
    """
    x = np.asarray(x, dtype=np.float64)
    f = x.astype(np.float32)
    if not np.array_equal(f.astype(np.float64), x, equal_nan=True):
        raise ValueError("value not representable in float32")
    u = f.view(np.uint32)
    if np.any(u & np.uint32(0xFFFF)):
        raise ValueError("value not representable in bf16")
    return (u >> np.uint32(16)).astype(np.uint16)
