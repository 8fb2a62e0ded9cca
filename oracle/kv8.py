"""FP8 main-KV rows: the compressed cache stored in 8-bit floats, the position-sensitive
dimensions kept in bf16 (test infrastructure: only tests/, the smoke check and the bench's CPU
baseline use this module).

[SW] shareware.cn/news/167317 §十三.4 (and §十四.4) says the main KV may be stored in FP8 while
the dimensions that are more sensitive to position information keep a higher precision; it
gives no format.  The reading taken here (plainest form consistent with the rest):

* A compressed row is K (128 dims) followed by V (128 dims), as everywhere in the library.
* K's last 64 dimensions are the position-encoded (RoPE) ones, the convention of the
  DeepSeek attention families, and stay bf16 (round to nearest even from the row's value).
* K's first 64 dimensions and all of V are OCP E4M3 codes, each group (the 64 K dims, the
  128 V dims) with its own scale: scale = amax / 448 over the group (1 for an all-zero
  group), code = E4M3(value / scale), ties to even, saturating at 448.
* Storage, 336 bytes a row: K codes (64 B) | K RoPE dims as bf16 (128 B) | V codes (128 B) |
  scale_k fp32 | scale_v fp32 | 8 zero bytes.  A decoded value is code x scale (exact), the
  RoPE dims the bf16 value.

Pinned by tests/test_oracle_kv8.py: hand-built rows with known bytes, exactly representable
inputs, the all-zero group, ties, saturation and the relative-error bound of E4M3."""

from __future__ import annotations

import numpy as np

from . import codecs

D = 128                 # head dim: K and V are 128 wide each
K_FP8 = 64              # K dims stored as E4M3 (dims 0..63)
K_ROPE = D - K_FP8      # K dims kept in bf16 (dims 64..127)
ROW_BYTES = 336
OFF_K, OFF_ROPE, OFF_V, OFF_SCALE = 0, 64, 192, 320
E4M3_MAX = 448.0


def group_scale_f64(x: np.ndarray) -> np.ndarray:
    """Scale of each row of a group [N, G]: amax / 448, 1 where the group is all zero."""
    amax = np.max(np.abs(np.asarray(x, dtype=np.float64)), axis=1)
    return np.where(amax > 0, amax / E4M3_MAX, 1.0)


def quantize_rows_f64(rows: np.ndarray):
    """K||V rows [N, 256] (any float dtype, read exactly) -> (k_codes [N, 64] uint8,
    rope [N, 64] bf16 bits uint16, v_codes [N, 128] uint8, scale_k [N], scale_v [N] float64),
    every step exact in float64 before the one rounding of each encoder."""
    r = np.asarray(rows, dtype=np.float64)
    k8, rope, v = r[:, :K_FP8], r[:, K_FP8:D], r[:, D:2 * D]
    s_k, s_v = group_scale_f64(k8), group_scale_f64(v)
    k_codes = codecs.e4m3_encode(k8 / s_k[:, None])
    v_codes = codecs.e4m3_encode(v / s_v[:, None])
    rope_bits = codecs.bf16_encode(rope)
    return k_codes, rope_bits, v_codes, s_k, s_v


def pack_rows(k_codes, rope_bits, v_codes, scale_k, scale_v) -> np.ndarray:
    """The 336-byte storage rows [N, 336] uint8 (scales stored as fp32, little-endian)."""
    n = np.asarray(k_codes).shape[0]
    out = np.zeros((n, ROW_BYTES), dtype=np.uint8)
    out[:, OFF_K:OFF_K + K_FP8] = np.asarray(k_codes, dtype=np.uint8)
    out[:, OFF_ROPE:OFF_ROPE + 2 * K_ROPE] = np.ascontiguousarray(
        np.asarray(rope_bits, dtype="<u2")).view(np.uint8).reshape(n, 2 * K_ROPE)
    out[:, OFF_V:OFF_V + D] = np.asarray(v_codes, dtype=np.uint8)
    sc = np.stack([np.asarray(scale_k, dtype="<f4"), np.asarray(scale_v, dtype="<f4")], axis=1)
    out[:, OFF_SCALE:OFF_SCALE + 8] = np.ascontiguousarray(sc).view(np.uint8).reshape(n, 8)
    return out


def decode_rows(buf: np.ndarray) -> np.ndarray:
    """Storage rows [N, 336] uint8 -> K||V values [N, 256] float64 (exact)."""
    b = np.ascontiguousarray(np.asarray(buf, dtype=np.uint8))
    n = b.shape[0]
    sc = b[:, OFF_SCALE:OFF_SCALE + 8].copy().view("<f4").reshape(n, 2).astype(np.float64)
    out = np.empty((n, 2 * D), dtype=np.float64)
    out[:, :K_FP8] = codecs.e4m3_decode(b[:, OFF_K:OFF_K + K_FP8]) * sc[:, :1]
    rope = b[:, OFF_ROPE:OFF_ROPE + 2 * K_ROPE].copy().view("<u2").reshape(n, K_ROPE)
    out[:, K_FP8:D] = codecs.bf16_decode(rope)
    out[:, D:] = codecs.e4m3_decode(b[:, OFF_V:OFF_V + D]) * sc[:, 1:]
    return out


def quantize_to_storage_f64(rows: np.ndarray) -> np.ndarray:
    """quantize_rows_f64 then pack_rows, with the scales rounded to fp32 for storage."""
    k, rope, v, s_k, s_v = quantize_rows_f64(rows)
    return pack_rows(k, rope, v, s_k.astype(np.float32), s_v.astype(np.float32))


def quotient_error_bound(rows: np.ndarray) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Bounds on an fp32 evaluation of the quantiser (the rows themselves exact in fp32):
    (tol_k [N, 64], tol_v [N, 128], tol_scale [N, 2]).

    With u = 2^-24, amax is exact, the scale amax / 448 takes one rounding (relative u) and
    the quotient value / scale one more: |q32 - q| <= |q| (u + u + u^2), so twice 2u|q| bounds
    the quotient, and u * scale the stored scale."""
    r = np.asarray(rows, dtype=np.float64)
    u = 2.0 ** -24
    s_k, s_v = group_scale_f64(r[:, :K_FP8]), group_scale_f64(r[:, D:])
    qk = np.abs(r[:, :K_FP8]) / s_k[:, None]
    qv = np.abs(r[:, D:]) / s_v[:, None]
    return 4 * u * qk, 4 * u * qv, np.stack([u * s_k, u * s_v], axis=1)
