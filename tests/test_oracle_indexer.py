"""Pins of the oracle's Lightning Indexer score, causal visibility and top-k:
the pages' worked examples, brute-force enumeration and constructed ties."""

import itertools
import json
import os

import numpy as np
import pytest

from oracle import attention, codecs, indexer

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_relu_per_head_worked_example():
    g = json.load(open(os.path.join(GOLD, "indexer_relu_example.json")))
    h1, h2 = g["head_scores"]
    q = np.array([[h1], [h2]], dtype=np.float64)       # two heads, one dim
    k = np.array([[1.0]])
    assert indexer.index_scores(q, k)[0] == g["relu_sum"]
    assert float((k @ q.T).sum()) == g["plain_sum"]      # what the plain sum would give


def test_scores_scales_and_head_weights():
    rng = np.random.default_rng(0)
    Hi, di, V = 3, 8, 50
    q = rng.standard_normal((Hi, di))
    k = rng.standard_normal((V, di))
    sq = rng.uniform(0.5, 2.0, Hi)
    sk = rng.uniform(0.5, 2.0, V)
    w = np.array([2.0, 0.0, 0.5])
    got = indexer.index_scores(q, k, sq, sk, w)
    for i in range(V):
        ref = 0.0
        for h in range(Hi):
            dot = sum(q[h, j] * k[i, j] for j in range(di))
            ref += w[h] * max(0.0, sq[h] * sk[i] * dot)
        assert abs(got[i] - ref) <= 1e-12 * (1 + abs(ref))
    # all heads negative -> score exactly 0
    assert indexer.index_scores(-np.abs(q), np.abs(k))[0] == 0.0


def test_causal_block24_example():
    g = json.load(open(os.path.join(GOLD, "causal_block24.json")))
    m, blk, p = g["ratio"], g["block"], g["query"]
    assert not indexer.entry_visible(blk, p, m)
    assert indexer.visible_entries(p, m) == blk            # blocks 0..23 only
    assert indexer.entry_visible(blk, g["block_visible_at"], m)
    assert indexer.visible_entries(g["block_visible_at"], m) == blk + 1
    win = attention.window_tokens(p, 128)
    for t in g["window_covers"]:
        assert t in win
    assert 99 not in win
    assert list(range(m * blk, m * blk + m)) == g["block_tokens"]


def test_visibility_edges():
    assert indexer.visible_entries(0, 4) == 0
    assert indexer.visible_entries(2, 4) == 0
    assert indexer.visible_entries(3, 4) == 1
    assert indexer.visible_entries(127, 128) == 1
    assert indexer.visible_entries(126, 128) == 0
    assert indexer.visible_entries((1 << 20) - 1, 4) == 262144


def _brute_topk(scores, k):
    """Best k-subset by score sum; among equal sums the lexicographically
    smallest sorted index vector (lower indices win ties)."""
    n = len(scores)
    kk = min(k, n)
    best, best_key = None, None
    for sub in itertools.combinations(range(n), kk):
        key = (-sum(scores[i] for i in sub), sub)
        if best_key is None or key < best_key:
            best, best_key = sub, key
    out = np.full(k, -1, dtype=np.int64)
    out[:kk] = best
    return out


@pytest.mark.parametrize("seed", range(40))
def test_topk_equals_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(0, 13))
    k = int(rng.integers(1, 6))
    # integer scores from a small range force many exact ties
    scores = rng.integers(0, 4, n).astype(np.float64)
    if seed % 3 == 0:
        scores = rng.standard_normal(n)
    got = indexer.topk_select(scores, k)
    assert np.array_equal(got, _brute_topk(list(scores), k))


def test_topk_padding_and_order():
    s = np.array([0.5, 0.9, 0.9, 0.1])
    assert list(indexer.topk_select(s, 2)) == [1, 2]
    assert list(indexer.topk_select(s, 3)) == [0, 1, 2]
    assert list(indexer.topk_select(s, 6)) == [0, 1, 2, 3, -1, -1]
    assert list(indexer.topk_select(np.zeros(0), 3)) == [-1, -1, -1]
    assert indexer.kth_score(s, 3) == 0.5
    # ties at the threshold go to the lower index
    t = np.array([1.0, 0.0, 1.0, 1.0, 2.0])
    assert list(indexer.topk_select(t, 3)) == [0, 2, 4]


def test_pool_keys_means_blocks_including_a_partial_one():
    # integer-valued tokens: every mean below is exact in fp32
    k = np.array([[1, -2], [2, 0], [3, 4], [6, 2],       # entry 0: mean (3, 1)
                  [5, 5], [5, 5], [5, 5], [5, 5],         # entry 1: identical tokens
                  [8, -8], [0, 2]], dtype=np.float32)     # entry 2: partial, two tokens
    got = indexer.pool_keys(k, 4)
    assert got.dtype == np.float32 and got.shape == (3, 2)
    assert np.array_equal(got, np.array([[3, 1], [5, 5], [4, -3]], dtype=np.float32))


def test_pool_keys_is_linear_and_sums_in_token_order():
    rng = np.random.default_rng(5)
    a = rng.standard_normal((12, 16)).astype(np.float32)
    # scaling by 2 is exact in fp32, so pooling commutes with it bit for bit
    assert np.array_equal(indexer.pool_keys(2 * a), 2 * indexer.pool_keys(a))
    # fp32 sum in token order, then one division
    blk = a[4:8]
    want = ((((blk[0] + blk[1]).astype(np.float32) + blk[2]).astype(np.float32) + blk[3]).astype(np.float32)
            / np.float32(4)).astype(np.float32)
    assert np.array_equal(indexer.pool_keys(a)[1], want)
    assert np.allclose(indexer.pool_keys(a), a.reshape(3, 4, 16).mean(axis=1), rtol=1e-6, atol=1e-6)


def test_quantize_keys_scale_and_error_bound():
    rng = np.random.default_rng(6)
    keys = rng.standard_normal((200, 64)).astype(np.float32)
    keys[7] = 0.0
    codes, scale = indexer.quantize_keys(keys)
    assert codes.dtype == np.uint8 and scale.dtype == np.float32
    assert scale[7] == 1.0 and np.all(codes[7] == 0)
    # the largest magnitude of every non-zero key lands on +-448 (code 0x7E / 0xFE)
    for i in (0, 1, 100):
        j = int(np.argmax(np.abs(keys[i])))
        assert codes[i, j] & 0x7F == 0x7E
        assert scale[i] == np.float32(np.abs(keys[i]).max() / np.float32(448))
    # decoded * scale is within half an E4M3 step: relative 2^-4 for normals, and an
    # absolute 2^-10 * scale below the smallest normal
    deq = codecs.e4m3_decode(codes) * scale[:, None].astype(np.float64)
    err = np.abs(deq - keys.astype(np.float64))
    bound = np.maximum(np.abs(keys) * 2.0 ** -4, 2.0 ** -10 * scale[:, None])
    assert np.all(err <= bound * (1 + 1e-6))


# ---- the exact (fp64) pooling definition and its fp32 error band


def _e4m3_table():
    """Every finite E4M3 code with its value (NaN codes left out)."""
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.uint8)
    return codes, codecs.e4m3_decode(codes)


def test_pool_f64_lands_on_printed_e4m3_values():
    g = json.load(open(os.path.join(GOLD, "e4m3_values.json")))
    vals = {int(c, 16): v for c, v in g["codes"].items() if c != "0x80"}
    key = np.array(list(vals.values()), dtype=np.float64)          # amax 448 -> scale 1
    offs = np.array([3.0, -1.0, -4.0, 2.0])                         # sum 0: the mean is the key
    for mult in (1.0, 2.0, 0.25):                                   # scales 1, 2, 1/4 (exact)
        tok = np.stack([mult * key + o * (1 if mult >= 1 else 0) for o in offs])
        mean = indexer.pool_keys_f64(tok, 4)
        assert np.array_equal(mean[0], mult * key)
        codes, scale = indexer.quantize_keys_f64(mean)
        assert scale[0] == mult * 448.0 / 448.0
        assert [int(c) for c in codes[0]] == list(vals.keys())


def test_pool_f64_integer_means_and_partial_block():
    k = np.array([[1, -2], [2, 0], [3, 4], [6, 2], [8, -8], [0, 2]], dtype=np.float64)
    assert np.array_equal(indexer.pool_keys_f64(k, 4), np.array([[3, 1], [4, -3]], dtype=np.float64))
    codes, scale = indexer.quantize_keys_f64(np.zeros((1, 4)))
    assert scale[0] == 1.0 and np.all(codes == 0)


def test_pool_f64_codes_are_the_nearest_e4m3_values_by_brute_force():
    table_c, table_v = _e4m3_table()
    rng = np.random.default_rng(11)
    tok = rng.standard_normal((4 * 40, 16)) / 8.0
    codes, scale = indexer.quantize_keys_f64(indexer.pool_keys_f64(tok, 4))
    key = indexer.pool_keys_f64(tok, 4)
    for i in range(key.shape[0]):
        for j in range(key.shape[1]):
            dist = np.abs(table_v * scale[i] - key[i, j])
            best = np.flatnonzero(dist == dist.min())
            # ties between two neighbours go to the even mantissa; +-0 are one value
            pick = [c for c in table_c[best] if c & 1 == 0] or list(table_c[best])
            want = codecs.e4m3_decode(np.array(pick[:1], dtype=np.uint8))[0]
            assert codecs.e4m3_decode(codes[i:i + 1, j])[0] == want, (i, j)


def test_fp32_restatement_stays_inside_the_error_band():
    rng = np.random.default_rng(12)
    tok = (rng.standard_normal((4 * 3000, 64)) / 8.0).astype(np.float32)
    # a few adversarial blocks: large tokens that cancel beside small ones
    tok[0:4, :8] = np.array([[1e4], [1.0], [-1e4], [0.5]], dtype=np.float32)
    tok[4:8, :8] = np.array([[3.0], [-3.0], [1e-3], [2e-3]], dtype=np.float32)
    t64 = tok.astype(np.float64)
    key64 = indexer.pool_keys_f64(t64, 4)
    c64, s64 = indexer.quantize_keys_f64(key64)
    tol_v, tol_s = indexer.quotient_error_bound(t64, 4)
    c32, s32 = indexer.quantize_keys(indexer.pool_keys(tok, 4))
    # the scale and the quotient of the fp32 steps lie inside the bounds
    assert np.all(np.abs(s32.astype(np.float64) - s64) <= tol_s)
    key32 = indexer.pool_keys(tok, 4)
    v32 = (key32 / s32[:, None]).astype(np.float32).astype(np.float64)
    v64 = key64 / s64[:, None]
    assert np.all(np.abs(v32 - v64) <= tol_v)
    # codes: equal to the exact ones outside the band, inside it between the codes of its ends
    lo = codecs.e4m3_decode(codecs.e4m3_encode(v64 - tol_v))
    hi = codecs.e4m3_decode(codecs.e4m3_encode(v64 + tol_v))
    d32 = codecs.e4m3_decode(c32)
    assert np.all((d32 >= lo) & (d32 <= hi))
    sure = lo == hi
    assert np.all(d32[sure] == codecs.e4m3_decode(c64)[sure])
    assert (~sure).mean() < 1e-3  # the band is narrow: a handful of elements


def test_error_band_catches_a_planted_off_by_one_code():
    # a code one step off where the band is a single code must fail the band check
    rng = np.random.default_rng(13)
    tok = rng.standard_normal((16, 64)) / 8.0
    key = indexer.pool_keys_f64(tok, 4)
    c64, s64 = indexer.quantize_keys_f64(key)
    tol_v, _ = indexer.quotient_error_bound(tok, 4)
    v64 = key / s64[:, None]
    lo = codecs.e4m3_decode(codecs.e4m3_encode(v64 - tol_v))
    hi = codecs.e4m3_decode(codecs.e4m3_encode(v64 + tol_v))
    bad = c64.copy()
    j = int(np.argmax((lo == hi)[0] & (np.abs(v64[0]) > 1.0)))
    bad[0, j] = bad[0, j] + 1 if bad[0, j] & 0x7F < 0x7E else bad[0, j] - 1
    d = codecs.e4m3_decode(bad)
    assert not np.all((d >= lo) & (d <= hi))
