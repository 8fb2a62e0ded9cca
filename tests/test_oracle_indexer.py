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
