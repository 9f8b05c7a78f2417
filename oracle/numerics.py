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


# ---------------------------------------------------------------- FP8 (e4m3)
# The FP8 deployment the pages report ("DiffusionGemma深度拆解" 性能数据: H100
# FP8; "谷歌DiffusionGemma" 引入扩散机制: the vLLM FP8 benchmark) stores the
# LM-head weights in 8-bit floating point. e4m3 ("fn" variant): 1 sign bit, 4
# exponent bits with bias 7, 3 mantissa bits; exponent field 0 holds the
# subnormals m/8 * 2^-6; S.1111.111 is NaN; no infinities; largest finite
# 448 = 1.75 * 2^8.
E4M3_MAX = 448.0


def _e4m3_value(b):
    """The value of e4m3 byte codes b (int64 array), from the format's definition."""
    sign = np.where((b & 0x80) != 0, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & (b & 7 == 7), np.nan, mag)
    return sign * mag


_E4M3_TABLE = _e4m3_value(np.arange(256, dtype=np.int64))  # the 256 codes' values


def e4m3_to_f64(codes):
    """e4m3 byte codes -> float64 (exact; a lookup in the table of the 256
    codes' values)."""
    return _E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


_E4M3_NONNEG = _E4M3_TABLE[:0x7F]  # codes 0..126, increasing


def round_to_e4m3(x):
    """float64 -> e4m3 byte codes, round to nearest with ties to the even code
    (the even mantissa). |x| must not exceed 448: callers scale into range, so
    no saturation rule is needed. The sign bit follows x (a negative value
    that rounds to zero gives the code of -0)."""
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.abs(x) <= E4M3_MAX):
        raise ValueError("value outside the e4m3 range")
    a = np.abs(x)
    hi = np.minimum(np.searchsorted(_E4M3_NONNEG, a, side="left"), 126)  # first value >= a
    lo = np.maximum(hi - 1, 0)
    dlo = a - _E4M3_NONNEG[lo]
    dhi = _E4M3_NONNEG[hi] - a
    pick = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo % 2 == 0, lo, hi)))
    pick = np.where(dhi == 0, hi, pick)
    return (pick.astype(np.uint8) | np.where(np.signbit(x), 0x80, 0).astype(np.uint8)).astype(np.uint8)


def e4m3_scale_exponent(amax):
    """The smallest integer e with 448 * 2^e >= amax (0 for amax = 0): the
    power-of-two scale that brings a row's largest magnitude into the e4m3
    range. With amax = f 2^k (f in [0.5, 1)) and 448 = 0.875 2^9 this is
    k - 9 when f <= 0.875, else k - 8 (exact integer arithmetic)."""
    amax = np.asarray(amax, dtype=np.float64)
    f, k = np.frexp(amax)
    e = np.where(f <= 0.875, k - 9, k - 8)
    return np.where(amax > 0, e, 0).astype(np.int64)


def quantize_rows_e4m3(x):
    """Each row of x as e4m3 codes times a power of two: e = the row's
    e4m3_scale_exponent, codes = round_to_e4m3(x * 2^-e) (the scaling is
    exact). Returns (codes [rows][n], e [rows])."""
    x = np.asarray(x, dtype=np.float64)
    e = e4m3_scale_exponent(np.max(np.abs(x), axis=-1))
    return round_to_e4m3(x * np.exp2(-e.astype(np.float64))[..., None]), e
