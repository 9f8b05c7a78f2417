"""Storage-format conversions used by the fp64 oracle.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

The GPU path stores a few intermediates (Q, canvas K/V, attention output O, the
residual stream Hs, the MoE expert intermediate) in the model's storage dtype.
The oracle computes every value in fp64 and rounds to that dtype at exactly
those points, with round-to-nearest-even.
"""
import numpy as np


def bf16_bits_to_f64(bits):
    """uint16 bf16 bit patterns -> float64 (exact: bf16 is the top half of fp32)."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def round_to_bf16(x):
    """Round float64 values to the nearest bf16 value (ties to even), returned as
    float64. Works on the fp64 bit pattern directly: bf16 keeps 7 explicit
    significand bits, fp64 has 52, so 45 bits are dropped; no intermediate
    rounding to fp32 happens. Values in the fp32 normal range only (the path's
    values are O(1e2) at most); inf/nan are passed through unchanged."""
    x = np.asarray(x, dtype=np.float64)
    bits = x.view(np.uint64).copy()
    finite = np.isfinite(x)
    drop = np.uint64(45)
    lsb = (bits >> drop) & np.uint64(1)
    half = np.uint64((1 << 44) - 1)
    rounded = (bits + half + lsb) >> drop << drop
    out = np.where(finite, rounded, bits).view(np.float64)
    return out


def round_to_f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_storage(x, dtype):
    """Round to the storage dtype: 'bf16' or 'f32'."""
    if dtype == "bf16":
        return round_to_bf16(x)
    if dtype == "f32":
        return round_to_f32(x)
    raise ValueError(dtype)


def widen(w, dtype):
    """Stored weights (uint16 bf16 bits or float32) -> float64. An array that is
    already float64 holds widened values and is returned unchanged."""
    if getattr(w, "dtype", None) == np.float64:
        return w
    if dtype == "bf16":
        return bf16_bits_to_f64(w)
    return np.asarray(w, dtype=np.float64)
