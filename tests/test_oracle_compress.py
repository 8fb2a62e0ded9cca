"""Pins of the oracle's CSA / HCA compression against what the pages fix and
against closed forms (mean pooling, one-hot weights, two-candidate softmax)."""

import json
import os

import numpy as np
import pytest

from oracle import compress

GOLD = os.path.join(os.path.dirname(__file__), "golden")
D = 256


def _rows(rng, n, scale=1.0):
    return rng.standard_normal((n, D)) * scale


def _csa(entries, n, xa, za, xb, zb, ba=None, bb=None):
    return compress.csa_compress(entries, n, xa, za, xb, zb, ba, bb)


def test_entry_counts_from_pages():
    g = json.load(open(os.path.join(GOLD, "entry_counts.json")))
    for c in g["cases"]:
        got = compress.num_entries(c["n"], c["ratio"])
        if "entries" in c:
            assert got == c["entries"]
        else:
            assert abs(got - c["entries_about"]) / c["entries_about"] < 0.01
    assert compress.num_entries(4099, 4) == 1025 and compress.num_entries(4096, 4) == 1024
    assert compress.num_entries(129, 128) == 2 and compress.num_entries(0, 4) == 0


def test_block_partition_from_pages():
    g = json.load(open(os.path.join(GOLD, "block_partition.json")))
    # one-hot logits pick exactly one token per entry: entry i must pick from tokens of block i
    n = 12
    rng = np.random.default_rng(0)
    xa = _rows(rng, n)
    for i, toks in enumerate(g["blocks"]):
        for slot, t in enumerate(toks):
            za = np.zeros((n, D))
            za[t] = 60.0
            zb = np.full((n, D), -np.inf)
            out = _csa([i], n, xa, za, xa, zb)
            np.testing.assert_allclose(out[0], xa[t], rtol=0, atol=1e-20)


def test_uniform_logits_single_path_is_mean_pooling():
    rng = np.random.default_rng(1)
    n = 40
    xa, xb = _rows(rng, n), _rows(rng, n)
    za = np.full((n, D), 0.7)
    zb = np.full((n, D), -np.inf)
    out = _csa(range(10), n, xa, za, xb, zb)
    ref = xa.reshape(10, 4, D).mean(axis=1)
    np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-15)


def test_uniform_logits_two_paths_is_mean_over_eight():
    rng = np.random.default_rng(2)
    n = 40
    xa, xb = _rows(rng, n), _rows(rng, n)
    z = np.full((n, D), -1.3)
    out = _csa(range(10), n, xa, z, xb, z)
    ref0 = xa[0:4].mean(axis=0)                                # entry 0: no previous block
    np.testing.assert_allclose(out[0], ref0, rtol=1e-13, atol=1e-15)
    for i in range(1, 10):
        ref = (xa[4 * i:4 * i + 4].sum(axis=0) + xb[4 * i - 4:4 * i].sum(axis=0)) / 8.0
        np.testing.assert_allclose(out[i], ref, rtol=1e-13, atol=1e-15)


def test_two_candidate_closed_form():
    # Block of one present token in path A (partial block) and ... use a 2-token HCA-like block:
    # logits (0, ln 3) give weights (1/4, 3/4).
    rng = np.random.default_rng(3)
    x = _rows(rng, 2)
    z = np.zeros((2, D))
    z[1] = np.log(3.0)
    out = compress.compress_entries([0], 2, 2, (x, z, None, 0))
    np.testing.assert_allclose(out[0], 0.25 * x[0] + 0.75 * x[1], rtol=1e-13, atol=1e-15)


def test_weights_are_per_dimension():
    # each dimension picks a different token: a per-token scalar weight could not do this
    rng = np.random.default_rng(4)
    n = 8
    xa, xb = _rows(rng, n), _rows(rng, n)
    za = np.zeros((n, D))
    zb = np.zeros((n, D))
    pick = rng.integers(0, 8, D)            # 0..3: path A slot of block 1; 4..7: path B slot of block 0
    ref = np.empty(D)
    for j, c in enumerate(pick):
        if c < 4:
            za[4 + c, j] = 80.0
            ref[j] = xa[4 + c, j]
        else:
            zb[c - 4, j] = 80.0
            ref[j] = xb[c - 4, j]
    out = _csa([1], n, xa, za, xb, zb)
    np.testing.assert_allclose(out[0], ref, rtol=0, atol=1e-30)


def test_dimension_permutation_commutes():
    rng = np.random.default_rng(5)
    n = 20
    xa, za, xb, zb = (_rows(rng, n) for _ in range(4))
    perm = rng.permutation(D)
    a = _csa(range(5), n, xa, za, xb, zb)
    b = _csa(range(5), n, xa[:, perm], za[:, perm], xb[:, perm], zb[:, perm])
    np.testing.assert_allclose(a[:, perm], b, rtol=1e-14, atol=0)


def test_logit_shift_invariance_and_bias_slots():
    rng = np.random.default_rng(6)
    n = 16
    xa, za, xb, zb = (_rows(rng, n) for _ in range(4))
    a = _csa(range(4), n, xa, za, xb, zb)
    b = _csa(range(4), n, xa, za + 5.0, xb, zb + 5.0)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-15)
    # a large bias on path-A slot 2 selects token 4i+2; on path-B slot 1 selects token 4(i-1)+1
    ba = np.zeros((4, D))
    ba[2, :128] = 90.0
    bb = np.zeros((4, D))
    bb[1, 128:] = 90.0
    out = _csa([2], n, xa, np.zeros((n, D)), xb, np.zeros((n, D)), ba, bb)
    np.testing.assert_allclose(out[0, :128], xa[10, :128], rtol=0, atol=1e-30)
    np.testing.assert_allclose(out[0, 128:], xb[5, 128:], rtol=0, atol=1e-30)


def test_path_b_masked_reduces_to_single_stream():
    rng = np.random.default_rng(7)
    n = 30
    xa, za, xb = _rows(rng, n), _rows(rng, n), _rows(rng, n)
    zb = np.full((n, D), -np.inf)
    a = _csa(range(8), n, xa, za, xb, zb)
    b = compress.compress_entries(range(8), 4, n, (xa, za, None, 0))
    np.testing.assert_allclose(a, b, rtol=1e-14, atol=0)


def test_path_a_masked_mixes_previous_block():
    rng = np.random.default_rng(8)
    n = 16
    xa, xb = _rows(rng, n), _rows(rng, n)
    za = np.zeros((n, D))
    za[8:12] = -np.inf                      # block 2's own tokens silenced
    zb = np.full((n, D), 0.25)
    out = _csa([2], n, xa, za, xb, zb)
    np.testing.assert_allclose(out[0], xb[4:8].mean(axis=0), rtol=1e-13, atol=1e-15)


def test_overlap_reach_of_token_three():
    # tokens 3 and 4 straddle the block-0 / block-1 boundary; token 3 reaches
    # entry 0 through path A and entry 1 through path B, and nothing else.
    rng = np.random.default_rng(9)
    n = 20
    xa, za, xb, zb = (_rows(rng, n) for _ in range(4))
    base = _csa(range(5), n, xa, za, xb, zb)
    xa2 = xa.copy()
    xa2[3] += 1.0
    d_a = np.abs(_csa(range(5), n, xa2, za, xb, zb) - base).max(axis=1)
    xb2 = xb.copy()
    xb2[3] += 1.0
    d_b = np.abs(_csa(range(5), n, xa, za, xb2, zb) - base).max(axis=1)
    assert d_a[0] > 0 and np.all(d_a[1:] == 0)
    assert d_b[1] > 0 and d_b[0] == 0 and np.all(d_b[2:] == 0)


def test_partial_last_block_uses_present_tokens():
    rng = np.random.default_rng(10)
    n = 14                                  # entries 0..3, entry 3 has tokens 12, 13 only
    xa, xb = _rows(rng, n), _rows(rng, n)
    z = np.zeros((n, D))
    out = _csa(range(4), n, xa, z, xb, z)
    ref = (xa[12:14].sum(axis=0) + xb[8:12].sum(axis=0)) / 6.0
    np.testing.assert_allclose(out[3], ref, rtol=1e-13, atol=1e-15)
    h = compress.hca_compress([0, 1], 130, _rows(rng, 130), np.zeros((130, D)))
    assert h.shape == (2, D)


def test_hca_mean_and_one_hot():
    rng = np.random.default_rng(11)
    n = 256
    x = _rows(rng, n)
    out = compress.hca_compress([0, 1], n, x, np.zeros((n, D)))
    np.testing.assert_allclose(out, x.reshape(2, 128, D).mean(axis=1), rtol=1e-13, atol=1e-15)
    z = np.zeros((n, D))
    z[128 + 77] = 100.0
    out = compress.hca_compress([1], n, x, z)
    np.testing.assert_allclose(out[0], x[128 + 77], rtol=0, atol=1e-30)
    bias = np.zeros((128, D))
    bias[5] = 100.0
    out = compress.hca_compress([0, 1], n, x, np.zeros((n, D)), bias)
    np.testing.assert_allclose(out, x[[5, 133]], rtol=0, atol=1e-30)


def test_tail_rows_offset():
    rng = np.random.default_rng(12)
    n = 40
    xa, za, xb, zb = (_rows(rng, n) for _ in range(4))
    full = _csa([8, 9], n, xa, za, xb, zb)
    t0 = 28
    tail = compress.csa_compress([8, 9], n, xa[t0:], za[t0:], xb[t0:], zb[t0:], tok0=t0)
    np.testing.assert_array_equal(full, tail)
    with pytest.raises(ValueError):
        compress.csa_compress([7], n, xa[t0:], za[t0:], xb[t0:], zb[t0:], tok0=t0)
