"""Pins of the oracle's storage codecs (bf16, OCP E4M3) against the format
specification's printed values and against torch's own conversions."""

import json
import os

import numpy as np
import pytest
import torch

from oracle import codecs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_e4m3_known_values_from_spec():
    g = json.load(open(os.path.join(GOLD, "e4m3_values.json")))
    for code, val in g["codes"].items():
        got = codecs.e4m3_decode(np.array([int(code, 16)], np.uint8))[0]
        assert got == val and np.signbit(got) == np.signbit(val), code
    for code in g["nan_codes"]:
        assert np.isnan(codecs.e4m3_decode(np.array([int(code, 16)], np.uint8))[0])


def test_e4m3_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = codecs.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])


def test_bf16_decode_matches_torch_all_codes():
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = codecs.bf16_decode(codes)
    ref = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])


@pytest.mark.parametrize("seed", [0, 1])
def test_bf16_encode_matches_torch_rne(seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-30, 30, 200000))).astype(np.float32)
    # exact halfway points between neighbouring bf16 values (ties go to even)
    # finite values only: the top 16 bits stay below the all-ones exponent
    base = rng.integers(0, 0x7F7F, 5000).astype(np.uint32) << np.uint32(16)
    half = (base | np.uint32(0x8000)).view(np.float32)
    # fp32 subnormals and values next to the overflow threshold
    sub = (rng.integers(1, 1 << 23, 2000).astype(np.uint32)).view(np.float32)
    big = np.array([3.3895314e38, 3.3961776e38, 3.4e38, -3.39e38, np.inf, -np.inf, 0.0, -0.0], np.float32)
    allx = np.concatenate([x, half, -half, sub, big])
    ours = codecs.bf16_encode(allx.astype(np.float64))
    ref = torch.from_numpy(allx).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_encode_rounds_doubles_once():
    # 1 + 2^-8 + 2^-30 lies just above the midpoint of 1 and 1 + 2^-7: it must round up,
    # while a detour through float32 (which drops the 2^-30) would tie to even and round down.
    x = np.array([1.0 + 2.0 ** -8 + 2.0 ** -30, 1.0 + 2.0 ** -8])
    got = codecs.bf16_decode(codecs.bf16_encode(x))
    assert got[0] == 1.0 + 2.0 ** -7
    assert got[1] == 1.0


def test_e4m3_encode_spec_values_and_nan():
    g = json.load(open(os.path.join(GOLD, "e4m3_values.json")))
    for code, val in g["codes"].items():
        assert codecs.e4m3_encode(np.array([val]))[0] == int(code, 16), code
    assert codecs.e4m3_encode(np.array([np.nan]))[0] == 0x7F


def test_e4m3_encode_round_trips_every_finite_code():
    codes = np.arange(256, dtype=np.uint8)
    vals = codecs.e4m3_decode(codes)
    fin = ~np.isnan(vals)
    assert np.array_equal(codecs.e4m3_encode(vals[fin]), codes[fin])


def test_e4m3_encode_ties_go_to_the_even_code():
    vals = codecs.e4m3_decode(np.arange(0x7F))
    mids = (vals[:-1] + vals[1:]) / 2           # exactly halfway between neighbours
    got = codecs.e4m3_encode(mids)
    lo = np.arange(0x7E)
    assert np.array_equal(got, np.where(lo % 2 == 0, lo, lo + 1))
    # just off the midpoint the nearer neighbour wins
    eps = (vals[1:] - vals[:-1]) / 64
    assert np.array_equal(codecs.e4m3_encode(mids - eps), lo)
    assert np.array_equal(codecs.e4m3_encode(mids + eps), lo + 1)


def test_e4m3_encode_saturates_and_keeps_sign():
    big = np.array([448.0, 449.0, 464.0, 480.0, 1e6, np.inf])
    assert np.all(codecs.e4m3_encode(big) == 0x7E)
    assert np.all(codecs.e4m3_encode(-big) == 0xFE)
    assert codecs.e4m3_encode(np.array([-1e-9]))[0] == 0x80   # rounds to -0
    assert codecs.e4m3_encode(np.array([2.0 ** -10]))[0] == 0x00  # half of the least subnormal: even (0)
    assert codecs.e4m3_encode(np.array([1.5 * 2.0 ** -9]))[0] == 0x02  # between 1 and 2 subnormal steps: even


@pytest.mark.parametrize("seed", range(3))
def test_e4m3_encode_matches_torch_cast_in_range(seed):
    rng = np.random.default_rng(seed)
    x = np.concatenate([rng.normal(0, 50, 50000), rng.normal(0, 0.01, 50000)]).astype(np.float32)
    x = np.clip(x, -448, 448)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codecs.e4m3_encode(x.astype(np.float64)), ref)


def _mx_gold():
    return json.load(open(os.path.join(GOLD, "mx_fp4_values.json")))


def test_e2m1_and_e8m0_values_from_spec():
    g = _mx_gold()
    for code, val in g["e2m1"].items():
        c = np.array([int(code, 16)], np.uint8)
        got = codecs.e2m1_decode(c)[0]
        assert got == val and np.signbit(got) == np.signbit(val), code
        assert codecs.e2m1_encode(np.array([val]))[0] == int(code, 16), code
    for code, val in g["e8m0"].items():
        assert codecs.e8m0_decode(np.array([int(code, 16)]))[0] == val, code
    assert np.isnan(codecs.e8m0_decode(np.array([int(g["e8m0_nan"], 16)]))[0])
    assert g["block_size"] == codecs.MX_BLOCK and g["e2m1_emax"] == codecs.E2M1_EMAX


def test_e2m1_encode_ties_even_and_saturation():
    # midpoints between neighbours go to the even code (the value with mantissa bit 0)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    assert list(codecs.e2m1_decode(codecs.e2m1_encode(mids))) == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    assert list(codecs.e2m1_decode(codecs.e2m1_encode(-mids))) == [-0.0, -1.0, -1.0, -2.0, -2.0, -4.0, -4.0]
    assert np.all(codecs.e2m1_encode(np.array([6.0, 6.5, 7.0, 100.0])) == 0x7)
    assert codecs.e2m1_encode(np.array([-1e-9]))[0] == 0x8
    # off the midpoints the nearer neighbour wins
    assert list(codecs.e2m1_decode(codecs.e2m1_encode(np.array([0.26, 2.49, 4.99, 5.01])))) == [0.5, 2.0, 4.0, 6.0]


def test_mx_fp4_shared_exponent_and_exact_powers_of_two():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((20, 64)) * np.ldexp(1.0, rng.integers(-20, 20, (20, 1)))
    codes, scales = codecs.mx_fp4_quantize(x)
    assert codes.shape == (20, 64) and scales.shape == (20, 2)
    amax = np.abs(x).reshape(20, 2, 32).max(axis=2)
    assert np.array_equal(scales.astype(np.int64) - 127, np.floor(np.log2(amax)).astype(np.int64) - 2)
    # the block maximum lands in [4, 6] times the scale (6 when it saturates)
    deq = codecs.mx_fp4_decode(codes, scales)
    top = np.abs(deq).reshape(20, 2, 32).max(axis=2) / codecs.e8m0_decode(scales)
    assert np.all((top >= 4.0) & (top <= 6.0))
    # blocks of representable magnitudes times one power of two come back exactly
    vals = codecs.e2m1_decode(rng.integers(0, 16, (5, 64)))
    vals[:, 0] = 6.0
    vals[:, 32] = -4.0
    y = vals * np.ldexp(1.0, 9)
    c2, s2 = codecs.mx_fp4_quantize(y)
    assert np.array_equal(codecs.mx_fp4_decode(c2, s2), y)


def test_mx_fp4_error_bound_and_zero_block():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((50, 64))
    x[3, :32] = 0.0
    codes, scales = codecs.mx_fp4_quantize(x)
    assert scales[3, 0] == 0 and np.all(codes[3, :32] == 0)
    X = np.repeat(codecs.e8m0_decode(scales), 32, axis=1)
    r = np.abs(x) / X
    deq = codecs.mx_fp4_decode(codes, scales)
    # half the E2M1 spacing at the element's magnitude; above 6 the element saturates to 6
    half = np.where(r < 2, 0.25, np.where(r < 4, 0.5, 1.0)) * X
    inside = r <= 6
    assert np.all(np.abs(deq - x)[inside] <= half[inside] * (1 + 1e-12))
    assert np.all(np.abs(deq[~inside]) == 6 * X[~inside])


def test_nibble_packing_order_and_round_trip():
    c = np.arange(16, dtype=np.uint8)
    p = codecs.pack_nibbles(c)
    assert list(p) == [0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE]
    assert np.array_equal(codecs.unpack_nibbles(p), c)
