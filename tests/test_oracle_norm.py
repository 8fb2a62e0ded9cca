"""Pins of the oracle's RMSNorm of queries and KV entries: closed forms, invariances, the
logit bound the pages want from it, and torch's rms_norm."""

import numpy as np
import pytest
import torch

from oracle import norm


def test_closed_form_example():
    y = norm.rmsnorm(np.array([3.0, 4.0]), eps=0.0)
    r = np.sqrt((9.0 + 16.0) / 2)
    assert np.allclose(y, [3.0 / r, 4.0 / r], rtol=0, atol=1e-15)


def test_unit_rms_scale_invariance_sign_and_gain():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((50, 128)) * rng.uniform(0.01, 100, (50, 1))
    y = norm.rmsnorm(x, eps=0.0)
    assert np.allclose(np.mean(y * y, axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.allclose(norm.rmsnorm(7.5 * x, eps=0.0), y, rtol=1e-13, atol=1e-13)
    assert np.array_equal(norm.rmsnorm(-x, eps=0.0), -y)
    g = rng.uniform(0.5, 2.0, 128)
    assert np.allclose(norm.rmsnorm(x, g, eps=0.0), y * g, rtol=1e-15, atol=1e-15)


def test_zero_vector_and_eps():
    assert np.array_equal(norm.rmsnorm(np.zeros(128), eps=1e-6), np.zeros(128))
    # eps only matters against tiny vectors: 1e-4 in every dimension -> 1e-4 / sqrt(1e-8 + 1e-6)
    y = norm.rmsnorm(np.full(4, 1e-4), eps=1e-6)
    assert np.allclose(y, 1e-4 / np.sqrt(1e-8 + 1e-6), rtol=1e-14)


def test_logits_are_bounded_after_normalisation():
    # unit gains: |q| = |k| = sqrt(d), so |<q, k>| <= d whatever the inputs' magnitudes,
    # with equality when k is a positive multiple of q
    rng = np.random.default_rng(1)
    d = 128
    q = norm.rmsnorm(rng.standard_normal((16, d)) * 1e3, eps=0.0)
    k = norm.rmsnorm(rng.standard_normal((64, d)) * 1e-3, eps=0.0)
    assert np.all(np.abs(q @ k.T) <= d * (1 + 1e-12))
    qq = norm.rmsnorm(q * 5.0, eps=0.0)
    assert np.allclose(np.sum(q * qq, axis=1), d, rtol=1e-12)


def test_packed_rows_normalise_each_half():
    rng = np.random.default_rng(2)
    rows = rng.standard_normal((10, 256))
    rows[:, 128:] *= 40.0
    out = norm.norm_packed_rows(rows, eps=0.0)
    assert np.allclose(np.mean(out[:, :128] ** 2, axis=1), 1.0, atol=1e-12)
    assert np.allclose(np.mean(out[:, 128:] ** 2, axis=1), 1.0, atol=1e-12)
    assert np.allclose(out[:, :128], norm.rmsnorm(rows[:, :128], eps=0.0), rtol=0, atol=0)


@pytest.mark.parametrize("eps", [1e-6, 1e-2])
def test_matches_torch_rms_norm(eps):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((32, 128))
    g = rng.uniform(0.5, 2.0, 128)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (128,), torch.from_numpy(g), eps=eps).numpy()
    assert np.allclose(norm.rmsnorm(x, g, eps), ref, rtol=1e-13, atol=1e-13)
