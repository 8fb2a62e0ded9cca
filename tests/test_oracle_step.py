"""End-to-end pins of the oracle's step on small synthetic workloads:
dense equivalence when k covers every visible entry, planted needles land in
the top-k, tail-row compression agrees with full-row compression."""

import math

import numpy as np
import pytest
import torch

from oracle import codecs, indexer, step
from synth import Workload, spec_by_name


def _np_arrays(w):
    return {k: w.numpy(k) for k in w.arrays}


def _dtypes(w):
    return {"kv": w.spec.dtype, "idx": w.spec.idx_dtype}


def _sdpa_dense(q, keys, values, sink, scale):
    """Textbook attention (torch, float64) of one query; sink = zero key + additive mask."""
    H, d = q.shape
    Q = torch.from_numpy(q)[None, :, None, :]
    K = torch.from_numpy(keys)[None, None].expand(1, H, -1, -1)
    V = torch.from_numpy(values)[None, None].expand(1, H, -1, -1)
    K = torch.cat([K, torch.zeros(1, H, 1, d, dtype=torch.float64)], dim=2)
    V = torch.cat([V, torch.zeros(1, H, 1, d, dtype=torch.float64)], dim=2)
    mask = torch.zeros(1, H, 1, K.shape[2], dtype=torch.float64)
    mask[..., -1] = torch.from_numpy(sink)[None, :, None]
    return torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask, scale=scale)[0, :, 0].numpy()


def test_tiny_dense_equivalence_when_k_covers_all():
    spec = spec_by_name("tiny").replace(seq_len=(700,), topk=4096)
    w = Workload(spec)
    m, a = w.meta, _np_arrays(w)
    res = step.run_step(m, a, _dtypes(w), bulk=True)
    p = m["q_pos"][0]
    V = indexer.visible_entries(p, 4)
    assert list(res["idx"][0][:V]) == list(range(V)) and np.all(res["idx"][0][V:] == -1)
    cmp = codecs.decode(res["cmp_c"][:V], "f32")
    raw = codecs.decode(a["raw_c"], "f32")
    toks = np.arange(max(0, p - 127), p + 1) - m["raw_t0"][0]
    rows = np.concatenate([cmp, raw[toks]])
    q = codecs.decode(a["q_c"][0], "f32")
    ref = _sdpa_dense(q, rows[:, :128], rows[:, 128:], a["sink_c"].astype(np.float64), m["scale"])
    np.testing.assert_allclose(res["o_c"][0], ref, rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(res["psink_c"][0], np.exp(a["sink_c"] - res["lse_c"][0]), rtol=1e-12)


def test_tiny_hca_dense_matches_textbook():
    w = Workload(spec_by_name("tiny_bias").replace(seq_len=(1000,)))
    m, a = w.meta, _np_arrays(w)
    res = step.run_step(m, a, _dtypes(w), bulk=True)
    p = m["q_pos"][0]
    vh = indexer.visible_entries(p, 128)
    cmp = codecs.decode(res["cmp_h"][:vh], "f32")
    raw = codecs.decode(a["raw_h"], "f32")
    toks = np.arange(max(0, p - 127), p + 1) - m["raw_t0"][0]
    rows = np.concatenate([cmp, raw[toks]])
    q = codecs.decode(a["q_h"][0], "f32")
    ref = _sdpa_dense(q, rows[:, :128], rows[:, 128:], a["sink_h"].astype(np.float64), m["scale"])
    np.testing.assert_allclose(res["o_h"][0], ref, rtol=1e-10, atol=1e-13)


def test_needles_are_selected():
    spec = spec_by_name("b1_ctx1m").replace(seq_len=(1 << 16,), heads=8)
    w = Workload(spec)
    assert len(w.needles) == 16
    m, a = w.meta, _np_arrays(w)
    s = step.query_scores(m, a, _dtypes(w), 0)
    sel = indexer.topk_select(s, m["k"])
    assert set(w.needles) <= set(sel.tolist())
    # the needles are far above the k-th score, not near-ties
    assert s[w.needles].min() > indexer.kth_score(s, m["k"]) + 0.1


def test_tail_compression_equals_full_compression():
    spec = spec_by_name("tiny").replace(seq_len=(1030,))
    full = Workload(spec)
    tail = Workload(spec.replace(cache="random"))
    m_f, a_f = full.meta, _np_arrays(full)
    m_t, a_t = tail.meta, _np_arrays(tail)
    assert m_t["csa_t0"][0] == 4 * (1029 // 4 - 1) and m_t["hca_t0"][0] == 1024
    # tails hold different random draws: build a full-row array set whose tail rows equal the tail draws
    a_mix = dict(a_f)
    for nm, t0 in (("x_a", "csa_t0"), ("z_a", "csa_t0"), ("x_b", "csa_t0"), ("z_b", "csa_t0"),
                   ("x_h", "hca_t0"), ("z_h", "hca_t0")):
        arr = a_f[nm].copy()
        arr[m_t[t0][0]:] = a_t[nm]
        a_mix[nm] = arr
    _, _, new_t = step.compress_step(m_t, a_t, _dtypes(tail))
    _, _, new_f = step.compress_step(m_f, a_mix, _dtypes(full), bulk=True)
    for layer in ("csa", "hca"):
        ents, rows = new_t[(layer, 0)]
        ents_f, rows_f = new_f[(layer, 0)]
        np.testing.assert_array_equal(rows, rows_f[ents])
    assert list(new_t[("csa", 0)][0]) == [257] and list(new_t[("hca", 0)][0]) == [8]


def test_prefill_queries_are_causal():
    spec = spec_by_name("prefill_4k_at_128k").replace(seq_len=(2048 + 64,), queries_per_seq=64, heads=4)
    w = Workload(spec)
    m, a = w.meta, _np_arrays(w)
    res = step.run_step(m, a, _dtypes(w), queries=[0, 1, 2, 3, 63])
    for j, t in enumerate(res["queries"]):
        p = m["q_pos"][t]
        V = indexer.visible_entries(p, 4)
        sel = res["idx"][j]
        assert np.all(sel[sel >= 0] < V)
        assert len(res["scores"][j]) == V
