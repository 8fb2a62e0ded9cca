"""GPU top-k selection, fed the oracle's fp32 scores: bit-exact against the
oracle's selection (ties to the lower index), across the kernel's paths:
single-CTA rows, multi-CTA groups with candidate compaction, the global
multi-pass path for massive ties, many-query row mode, padding."""

import numpy as np
import pytest
import torch

from oracle import indexer

from compressed_sparse_kv_compress_b200 import api

pytestmark = pytest.mark.gpu

_WS = {}


def _run(scores_rows, k, ld=None):
    T = len(scores_rows)
    ld = ld or max(1, max(len(s) for s in scores_rows))
    S = np.zeros((T, ld), np.float32)
    for t, s in enumerate(scores_rows):
        S[t, :len(s)] = s
    n = torch.tensor([len(s) for s in scores_rows], dtype=torch.int64, device="cuda")
    dev_s = torch.from_numpy(S).cuda()
    maxe = max(len(s) for s in scores_rows)
    key = (T, k, maxe)
    if key not in _WS:  # reused across calls: every call must leave it reusable
        _WS[key] = api.lindex_workspace(T, k, maxe)
    ws = _WS[key]
    out = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    osc = torch.empty(T, k, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.lindex_topk_from_scores(dev_s, n, out, ws, max_entries=maxe, out_score=osc, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return out.cpu().numpy(), osc.cpu().numpy()


def _check(rows, k, ld=None):
    out, osc = _run(rows, k, ld)
    for t, s in enumerate(rows):
        ref = indexer.topk_select(np.asarray(s, np.float32).astype(np.float64), k)
        assert np.array_equal(out[t], ref), f"row {t}: first mismatch at {np.nonzero(out[t] != ref)[0][:5]}"
        kk = min(k, len(s))
        assert np.array_equal(osc[t, :kk], np.asarray(s, np.float32)[ref[:kk]])


@pytest.mark.parametrize("V,k", [(1000, 64), (4096, 1024), (262144, 1024), (70000, 2048), (16384, 1024)])
def test_random_scores_single_query(V, k):
    rng = np.random.default_rng(V)
    _check([rng.standard_normal(V).astype(np.float32) * 0.2 + 0.4], k)


def test_relu_like_scores_with_zero_pile():
    rng = np.random.default_rng(1)
    s = np.maximum(rng.standard_normal((8, 65536)), 0).sum(axis=0).astype(np.float32)
    _check([s], 1024)
    _check([np.maximum(rng.standard_normal(3000), 0).astype(np.float32)], 2048)  # threshold lands on 0


def test_integer_ties_across_segments():
    rng = np.random.default_rng(2)
    _check([rng.integers(0, 50, 200000).astype(np.float32)], 1024)
    _check([rng.integers(0, 3, 50000).astype(np.float32)], 777)


def test_all_equal_scores_take_lowest_indices():
    _check([np.full(300000, 0.25, np.float32)], 1024)
    _check([np.full(5000, -1.5, np.float32)], 100)


def test_threshold_bin_overflow_uses_global_passes():
    # all scores share their top 12 key bits: the candidate set is too large to compact
    rng = np.random.default_rng(3)
    s = (1.0 + rng.random(200000) * 1e-3).astype(np.float32)
    _check([s], 1024)


def test_negative_zero_ranks_with_zero():
    s = np.array([0.0, -0.0, 1.0, -0.0, 0.0, -1.0] * 50, np.float32)
    _check([s], 120)


def test_padding_and_empty_rows():
    rng = np.random.default_rng(4)
    rows = [rng.random(10).astype(np.float32), np.zeros(0, np.float32), rng.random(1024).astype(np.float32),
            rng.random(1025).astype(np.float32)]
    _check(rows, 1024, ld=2048)


@pytest.mark.parametrize("T", [8, 64, 300])
def test_many_queries_ragged(T):
    rng = np.random.default_rng(T)
    rows = [rng.standard_normal(int(rng.integers(0, 40000))).astype(np.float32) for _ in range(T)]
    _check(rows, 512)


def test_repeated_calls_reuse_workspace():
    # the same workspace serves calls that take the speculative, the exact and the
    # single-CTA paths one after another
    rng = np.random.default_rng(5)
    rows_a = [rng.standard_normal(100000).astype(np.float32), rng.standard_normal(50000).astype(np.float32)]
    rows_b = [np.arange(100000, dtype=np.float32), np.full(50000, 2.0, np.float32)]
    for i in range(3):
        _check(rows_a, 1024)
        _check(rows_b, 1024)


def test_winners_concentrated_in_one_segment():
    # ascending scores put the whole top-k in the last segment of the group, so the
    # speculative proposals cannot cover it and the exact path must take over
    _check([np.arange(262144, dtype=np.float32)], 1024)
    s = np.random.default_rng(6).random(100000).astype(np.float32)
    s[40000:41500] += 10.0
    _check([s], 1024)
    _check([s[::-1].copy()], 1500)
