"""Storage formats, decoded and encoded exactly (oracle side).

* bf16: the upper 16 bits of an IEEE-754 binary32 (1 sign, 8 exponent,
  7 fraction bits).  Decoding shifts the code into the high half of a
  binary32, which is exact.  Encoding rounds a float64 straight to the
  nearest bf16 value, ties to even, overflowing to infinity.
* MXFP4: the OCP Microscaling format with E2M1 elements (1 sign, 2 exponent
  bits with bias 1, 1 mantissa bit: 0, 0.5, 1, 1.5, 2, 3, 4, 6) and one E8M0
  power-of-two scale per 32 elements; the pages name FP4 for the indexer's QK
  path without the variant, and this is the one sm_100 tensor cores take
  block-scaled (kind::mxf4).
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


# ---- MXFP4 (OCP Microscaling Formats v1.0): E2M1 elements, one E8M0 scale per 32
#      (the FP4 the pages name for the indexer's QK path: [SW] §六.1, §十三.4; [TR] §4.2)
E2M1_EMAX = 2        # exponent of the largest normal, 6 = 1.5 * 2^2
MX_BLOCK = 32


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """4-bit E2M1 codes (0..15) -> float64: sign bit 3, exponent bits 2..1 (bias 1),
    mantissa bit 0; exponent field 0 is the subnormal 0.5 * m."""
    c = np.asarray(codes, dtype=np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = (c & 0x1).astype(np.float64)
    mag = np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * np.ldexp(1.0, e - 1))
    return sign * mag


def e2m1_encode(x: np.ndarray) -> np.ndarray:
    """float64 -> E2M1 codes: nearest value, ties to the even code, magnitudes above 6
    saturating to 6, sign kept (-0 -> 0x8).  NaN is not representable (inputs finite)."""
    x = np.asarray(x, dtype=np.float64)
    table = e2m1_decode(np.arange(8))                 # 0, 0.5, 1, 1.5, 2, 3, 4, 6
    a = np.minimum(np.abs(x), 6.0)
    hi = np.clip(np.searchsorted(table, a, side="left"), 0, 7)
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - table[lo], table[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    return np.where(np.signbit(x), code | np.uint8(0x8), code).astype(np.uint8)


def e8m0_decode(codes: np.ndarray) -> np.ndarray:
    """E8M0 scale codes -> float64: 2^(code - 127); 0xFF is NaN."""
    c = np.asarray(codes, dtype=np.int64)
    return np.where(c == 0xFF, np.nan, np.ldexp(1.0, c - 127))


def mx_fp4_quantize(x: np.ndarray, block: int = MX_BLOCK) -> tuple[np.ndarray, np.ndarray]:
    """Values [..., n] (n a multiple of `block`) -> (E2M1 codes [..., n], E8M0 scale codes
    [..., n / block]) by the MX conversion: per block, shared exponent
    floor(log2(max |v|)) - E2M1_EMAX clamped to [-127, 127] (an all-zero block takes the
    smallest scale, 2^-127), then every element v / 2^shared converted to E2M1 (nearest
    even, saturating).  Dividing by a power of two is exact, so the codes do not depend on
    the precision the division is carried out in."""
    v = np.asarray(x, dtype=np.float64)
    shp = v.shape
    vb = v.reshape(shp[:-1] + (shp[-1] // block, block))
    amax = np.max(np.abs(vb), axis=-1)
    _, e2 = np.frexp(np.where(amax > 0, amax, 1.0))   # amax = f * 2^e2, f in [0.5, 1)
    shared = np.where(amax > 0, e2 - 1 - E2M1_EMAX, -127)
    shared = np.clip(shared, -127, 127)
    codes = e2m1_encode(vb / np.ldexp(1.0, shared)[..., None])
    return codes.reshape(shp), (shared + 127).astype(np.uint8)


def mx_fp4_decode(codes: np.ndarray, scales: np.ndarray, block: int = MX_BLOCK) -> np.ndarray:
    """E2M1 codes [..., n] and E8M0 scales [..., n / block] -> float64 values."""
    c = np.asarray(codes)
    shp = c.shape
    vals = e2m1_decode(c).reshape(shp[:-1] + (shp[-1] // block, block))
    return (vals * e8m0_decode(scales)[..., None]).reshape(shp)


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """4-bit codes [..., n] (n even) -> bytes [..., n / 2]: element 2j in the low nibble of
    byte j, element 2j + 1 in the high nibble."""
    c = np.asarray(codes, dtype=np.uint8) & 0xF
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    """Inverse of pack_nibbles."""
    b = np.asarray(packed, dtype=np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out


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
