"""Storage formats, decoded and encoded exactly (oracle side).

* bf16: the upper 16 bits of an IEEE-754 binary32 (1 sign, 8 exponent,
  7 fraction bits).  Decoding shifts the code into the high half of a
  binary32, which is exact.  Encoding rounds a float64 straight to the
  nearest bf16 value, ties to even, overflowing to infinity.
* E4M3: the OCP 8-bit floating point format (1 sign, 4 exponent bits with
  bias 7, 3 mantissa bits; exponent field 0 holds subnormals 2^-6 * m/8;
  no infinities; S.1111.111 is NaN; largest finite value 448).  The pages
  name FP8 for the indexer's QK path ([SW] §六.1 and §十三.4; [TR] §4.2
  "linear_fp8", "FP8或者FP4"), but not which FP8 variant; E4M3 is the
  variant with the finer mantissa and is the one used here.
"""

from __future__ import annotations

import numpy as np


def bf16_decode(codes: np.ndarray) -> np.ndarray:
    """uint16 bf16 codes -> float64 (exact)."""
    c = np.asarray(codes, dtype=np.uint16)
    with np.errstate(invalid="ignore"):
        return (c.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def bf16_encode(x: np.ndarray) -> np.ndarray:
    """float64 -> uint16 bf16 codes, round to nearest, ties to even."""
    x = np.asarray(x, dtype=np.float64)
    sign = np.signbit(x)
    a = np.abs(x)
    out = np.zeros(x.shape, dtype=np.float64)
    fin = np.isfinite(a) & (a > 0)
    if np.any(fin):
        _, e2 = np.frexp(a[fin])           # a = f * 2^e2, f in [0.5, 1)
        e = np.maximum(e2 - 1, -126)       # unbiased exponent, clamped to the normal range
        q = np.ldexp(1.0, e - 7)           # spacing of bf16 values at this exponent
        out[fin] = np.rint(a[fin] / q) * q  # np.rint rounds half to even
    out[np.isinf(a)] = np.inf
    out = np.where(out >= 2.0 ** 128, np.inf, out)
    with np.errstate(invalid="ignore", over="ignore"):
        bits = (out.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    bits = np.where(sign & ~np.isnan(x), bits | np.uint16(0x8000), bits)
    bits = np.where(np.isnan(x), np.uint16(0x7FC0), bits)
    return bits.astype(np.uint16)


def f32_encode(x: np.ndarray) -> np.ndarray:
    """float64 -> float32, round to nearest even (numpy's cast)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """uint8 OCP E4M3 codes -> float64 (exact; NaN for S.1111.111)."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.ldexp(1.0, e - 7))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """float64 -> uint8 OCP E4M3 codes: the nearest finite E4M3 value, ties to the even
    code (the one whose mantissa's last bit is 0), magnitudes above 448 saturating to 448;
    the sign is kept, zero results included (-0 -> 0x80); NaN -> 0x7F.

    The positive finite values are those of codes 0x00..0x7E, ascending with the code, so
    the encoding is a nearest-neighbour search in that table."""
    x = np.asarray(x, dtype=np.float64)
    table = e4m3_decode(np.arange(0x7F))            # 0, 2^-9, ..., 448 (ascending)
    a = np.minimum(np.abs(x), 448.0)
    hi = np.clip(np.searchsorted(table, a, side="left"), 0, 0x7E)   # first value >= a
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - table[lo], table[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(np.signbit(x), code | np.uint8(0x80), code).astype(np.uint8)
    return np.where(np.isnan(x), np.uint8(0x7F), code).astype(np.uint8)


def decode(arr: np.ndarray | None, dtype: str) -> np.ndarray | None:
    """Storage array -> float64.  dtype in {'bf16', 'f32', 'fp8'}."""
    if arr is None:
        return None
    if dtype == "bf16":
        return bf16_decode(arr)
    if dtype == "f32":
        return np.asarray(arr, dtype=np.float32).astype(np.float64)
    if dtype == "fp8":
        return e4m3_decode(arr)
    raise ValueError(dtype)


def encode(x: np.ndarray, dtype: str) -> np.ndarray:
    """float64 -> storage array (bf16 codes or float32)."""
    if dtype == "bf16":
        return bf16_encode(x)
    if dtype == "f32":
        return f32_encode(x)
    raise ValueError(dtype)
