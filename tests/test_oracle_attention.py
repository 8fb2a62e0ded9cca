"""Pins of the oracle's hybrid attention: probability mass with the sink, the
pages' 0.15 / 0.85 sink example, MQA == library attention with the KV head
repeated (GQA with one group), split-and-merge == one shot."""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _qkv(rng, H, N, d):
    return rng.standard_normal((H, d)), rng.standard_normal((N, d)), rng.standard_normal((N, d))


def test_probabilities_with_sink_sum_to_one():
    rng = np.random.default_rng(0)
    q, k, v = _qkv(rng, 8, 37, 16)
    sink = rng.standard_normal(8)
    o, lse, p, ps = attention.attend(q, k, v, sink, 0.25)
    np.testing.assert_allclose(p.sum(axis=1) + ps, 1.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(ps, np.exp(sink - lse), rtol=1e-12)
    # without a sink the real rows carry everything
    _, _, p2, ps2 = attention.attend(q, k, v, None, 0.25)
    np.testing.assert_allclose(p2.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(ps2 == 0)


def test_sink_example_from_pages():
    g = json.load(open(os.path.join(GOLD, "sink_example.json")))
    N, H, d = 50, 4, 8
    q = np.zeros((H, d))                         # every real logit is 0
    k = np.ones((N, d))
    v = np.random.default_rng(1).standard_normal((N, d))
    sigma = math.log(N * g["sink_mass"] / g["real_mass"])
    o, lse, p, ps = attention.attend(q, k, v, np.full(H, sigma), 1.0)
    np.testing.assert_allclose(ps, g["sink_mass"], rtol=1e-12)
    np.testing.assert_allclose(p.sum(axis=1), g["real_mass"], rtol=1e-12)
    np.testing.assert_allclose(o, np.tile(g["real_mass"] * v.mean(axis=0), (H, 1)), rtol=1e-12)


@pytest.mark.parametrize("with_sink", [False, True])
def test_mqa_equals_library_attention_with_repeated_kv(with_sink):
    rng = np.random.default_rng(2)
    H, N, d = 6, 29, 32
    q, k, v = _qkv(rng, H, N, d)
    sink = rng.standard_normal(H) if with_sink else None
    scale = 1.0 / math.sqrt(d)
    o, lse, _, _ = attention.attend(q, k, v, sink, scale)
    # GQA with one KV group: repeat the single KV head for every query head,
    # run the library's attention; the sink becomes one extra all-zero key whose
    # additive mask is sigma_h, and whose value row is zero.
    Q = torch.from_numpy(q)[None, :, None, :]                     # [1, H, 1, d]
    K = torch.from_numpy(k)[None, None].repeat_interleave(H, dim=1)
    V = torch.from_numpy(v)[None, None].repeat_interleave(H, dim=1)
    mask = torch.zeros(1, H, 1, N, dtype=torch.float64)
    if with_sink:
        K = torch.cat([K, torch.zeros(1, H, 1, d, dtype=torch.float64)], dim=2)
        V = torch.cat([V, torch.zeros(1, H, 1, d, dtype=torch.float64)], dim=2)
        mask = torch.cat([mask, torch.from_numpy(sink)[None, :, None, None]], dim=3)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask, scale=scale)
    np.testing.assert_allclose(o, ref[0, :, 0].numpy(), rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("seed", range(5))
def test_split_merge_equals_one_shot(seed):
    rng = np.random.default_rng(seed)
    H, N, d = 5, 61, 16
    q, k, v = _qkv(rng, H, N, d)
    q *= 3.0
    sink = rng.standard_normal(H) * 2 if seed % 2 else None
    o, lse, _, _ = attention.attend(q, k, v, sink, 0.5)
    cuts = np.sort(rng.choice(np.arange(1, N), size=int(rng.integers(1, 8)), replace=False))
    parts = [attention.partial(q, k[a:b], v[a:b], 0.5) for a, b in zip([0, *cuts], [*cuts, N])]
    o2, lse2 = attention.merge_partials(parts, sink)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse2, lse, rtol=1e-12)


def test_window_tokens_and_gather():
    assert list(attention.window_tokens(5, 128)) == list(range(6))
    assert list(attention.window_tokens(300, 128)) == list(range(173, 301))
    d = 4
    cmp_rows = np.arange(5 * 2 * d, dtype=np.float64).reshape(5, 2 * d)
    raw = -np.arange(10 * 2 * d, dtype=np.float64).reshape(10, 2 * d)
    keys, values = attention.gather_rows(cmp_rows, [1, 3], raw, 100, 104, 3, d)
    np.testing.assert_array_equal(keys[:2], cmp_rows[[1, 3], :d])
    np.testing.assert_array_equal(values[2:], raw[[2, 3, 4], d:])
    with pytest.raises(ValueError):
        attention.gather_rows(cmp_rows, [], raw, 100, 101, 3, d)


def test_empty_rows_with_sink_only():
    o, lse, p, ps = attention.attend(np.ones((2, 4)), np.zeros((0, 4)), np.zeros((0, 4)), np.array([0.3, -1.0]))
    np.testing.assert_allclose(ps, 1.0)
    np.testing.assert_array_equal(o, 0.0)
