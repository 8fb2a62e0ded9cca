"""Pins of oracle/kv8.py (FP8 main-KV rows, [SW] §十三.4) against values fixed by the OCP E4M3
and bf16 formats and by the row layout, not by the oracle's own arithmetic."""

import numpy as np

from oracle import codecs, kv8


def test_hand_built_row_decodes_to_known_values():
    # bytes written by hand at the documented offsets: E4M3 0x38 = 1.0, 0x40 = 2.0, 0xC0 = -2.0,
    # 0x01 = 2^-9 (smallest subnormal); bf16 0x3F80 = 1.0, 0xC040 = -3.0
    row = np.zeros((1, 336), dtype=np.uint8)
    row[0, 0] = 0x38            # K dim 0
    row[0, 63] = 0x40           # K dim 63
    row[0, 64:66] = [0x80, 0x3F]  # K dim 64 (first RoPE dim), little-endian bf16
    row[0, 190:192] = [0x40, 0xC0]  # K dim 127
    row[0, 192] = 0x01          # V dim 0
    row[0, 319] = 0xC0          # V dim 127
    row[0, 320:324] = np.frombuffer(np.float32(0.5).tobytes(), np.uint8)   # scale_k
    row[0, 324:328] = np.frombuffer(np.float32(4.0).tobytes(), np.uint8)   # scale_v
    x = kv8.decode_rows(row)[0]
    assert x[0] == 0.5 and x[63] == 1.0
    assert x[64] == 1.0 and x[127] == -3.0
    assert x[128] == 4.0 * 2.0 ** -9 and x[255] == -8.0
    assert np.count_nonzero(x) == 6


def test_exactly_representable_rows_round_trip():
    # K and V groups made of E4M3 values times a power of two, each group holding +-448 x that
    # power (so amax / 448 is the power itself): quantising must give back the same codes
    rng = np.random.default_rng(3)
    n = 32
    ck = rng.integers(0, 0x7F, (n, 64)).astype(np.uint8) | (rng.integers(0, 2, (n, 64)) << 7).astype(np.uint8)
    cv = rng.integers(0, 0x7F, (n, 128)).astype(np.uint8) | (rng.integers(0, 2, (n, 128)) << 7).astype(np.uint8)
    ck[:, 5] = 0x7E  # 448
    cv[:, 9] = 0xFE  # -448
    pk = 2.0 ** rng.integers(-12, 6, n)
    pv = 2.0 ** rng.integers(-12, 6, n)
    rope = rng.standard_normal((n, 64))
    rows = np.concatenate([codecs.e4m3_decode(ck) * pk[:, None], rope, codecs.e4m3_decode(cv) * pv[:, None]], axis=1)
    k, rb, v, s_k, s_v = kv8.quantize_rows_f64(rows)
    assert np.array_equal(s_k, pk) and np.array_equal(s_v, pv)
    # -0 and +0 decode alike; compare values
    assert np.array_equal(codecs.e4m3_decode(k), codecs.e4m3_decode(ck))
    assert np.array_equal(codecs.e4m3_decode(v), codecs.e4m3_decode(cv))
    got = kv8.decode_rows(kv8.pack_rows(k, rb, v, s_k.astype(np.float32), s_v.astype(np.float32)))
    assert np.array_equal(got[:, :64], rows[:, :64]) and np.array_equal(got[:, 128:], rows[:, 128:])
    # the RoPE dims: bf16 round to nearest even of the row's values
    assert np.array_equal(got[:, 64:128], codecs.bf16_decode(codecs.bf16_encode(rope)))


def test_bf16_rope_dims_are_kept_exactly():
    rng = np.random.default_rng(4)
    bits = rng.integers(0, 0x7F80, (8, 64)).astype(np.uint16)   # finite positive bf16
    rope = codecs.bf16_decode(bits)
    rows = np.concatenate([rng.standard_normal((8, 64)), rope, rng.standard_normal((8, 128))], axis=1)
    got = kv8.decode_rows(kv8.quantize_to_storage_f64(rows))
    assert np.array_equal(got[:, 64:128], rope)


def test_all_zero_group_has_scale_one_and_zero_codes():
    rows = np.zeros((2, 256))
    rows[1, 128:] = np.linspace(-1, 1, 128)   # row 1: K all zero, V not
    k, _, v, s_k, s_v = kv8.quantize_rows_f64(rows)
    assert np.all(s_k == 1.0) and s_v[0] == 1.0 and s_v[1] == 1.0 / 448.0
    assert np.all(codecs.e4m3_decode(k) == 0) and np.all(codecs.e4m3_decode(v[0]) == 0)
    assert np.array_equal(kv8.decode_rows(kv8.quantize_to_storage_f64(rows))[0], np.zeros(256))


def test_ties_go_to_even_code_and_amax_maps_to_448():
    # group amax 448 -> scale 1; 1.0625 lies half-way between 1.0 (0x38) and 1.125 (0x39):
    # ties to the even code 0x38; 1.1875 between 1.125 (0x39) and 1.25 (0x3A): 0x3A
    rows = np.zeros((1, 256))
    rows[0, 0], rows[0, 1], rows[0, 2] = 448.0, 1.0625, 1.1875
    rows[0, 128] = -448.0
    k, _, v, s_k, s_v = kv8.quantize_rows_f64(rows)
    assert s_k[0] == 1.0 and s_v[0] == 1.0
    assert k[0, 0] == 0x7E and k[0, 1] == 0x38 and k[0, 2] == 0x3A and v[0, 0] == 0xFE


def test_relative_error_within_half_an_e4m3_step():
    # normal E4M3 values carry 3 mantissa bits: rounding moves a value by at most 2^-4 of it;
    # below 2^-6 x scale (subnormals) by at most half the subnormal spacing 2^-10 x scale
    rng = np.random.default_rng(5)
    rows = rng.standard_normal((64, 256)) * np.exp(rng.uniform(-6, 6, (64, 1)))
    got = kv8.decode_rows(kv8.quantize_to_storage_f64(rows))
    for lo, hi in ((0, 64), (128, 256)):
        x = rows[:, lo:hi]
        s = np.max(np.abs(x), axis=1, keepdims=True) / 448.0
        s32 = s.astype(np.float32).astype(np.float64)
        # the stored scale is fp32: decode uses it, so compare against codes x the fp32 scale
        err = np.abs(got[:, lo:hi] - x)
        bound = np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * s) + np.abs(s32 - s) * 448.0
        assert np.all(err <= bound * (1 + 1e-12))
