"""GPU Lightning Indexer (scan + top-k in one call) against the oracle:
scores of the kept entries, and a selection that may differ from the oracle's
only for entries whose oracle score lies within 1e-4 of the k-th score."""

import numpy as np
import pytest
import torch

from oracle import step as ostep
from synth import Workload, spec_by_name

from compressed_sparse_kv_compress_b200 import api
from helpers import bounds, check_selection, dtypes, np_arrays

pytestmark = pytest.mark.gpu


def _run_indexer(w, dev=None):
    dev = dev or w.device("cuda")
    m = w.meta
    b = bounds(w)
    T, k = m["T"], m["k"]
    ws = api.lindex_workspace(T, k, b["max_csa_visible"])
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    sc = torch.empty(T, k, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.lindex_score_topk(dev["q_idx"], dev["k_idx"], dev["q_seq"], dev["q_pos"], dev["csa_off"], idx, ws,
                          max_entries=b["max_csa_visible"], q_scale=dev["q_scale"], k_scale=dev["k_scale"],
                          head_w=dev["head_w"], out_score=sc, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    first, first_sc = idx.clone(), sc.clone()
    # a second call on the same workspace gives the same selection; it also asks for the L2
    # prefetch of the kept rows of the compressed cache, a hint that changes no result
    api.lindex_score_topk(dev["q_idx"], dev["k_idx"], dev["q_seq"], dev["q_pos"], dev["csa_off"], idx, ws,
                          max_entries=b["max_csa_visible"], q_scale=dev["q_scale"], k_scale=dev["k_scale"],
                          head_w=dev["head_w"], out_score=sc, prefetch_rows=dev["cmp_c"], dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(first, idx) and torch.equal(first_sc, sc)
    return idx.cpu().numpy(), sc.cpu().numpy()


def _check_queries(w, queries, idx, sc):
    a = np_arrays(w)
    for t in queries:
        s = ostep.query_scores(w.meta, a, dtypes(w), t)
        check_selection(idx[t], s, w.meta["k"], f"query {t}")
        kk = min(w.meta["k"], len(s))
        sel = idx[t, :kk]
        err = np.abs(sc[t, :kk] - s[sel])
        assert err.max(initial=0) <= 1e-5 * max(1.0, np.abs(s).max(initial=0)), f"query {t}: score error"


def test_tiny_fp32():
    w = Workload(spec_by_name("tiny"))
    idx, sc = _run_indexer(w)
    _check_queries(w, [0], idx, sc)


@pytest.mark.parametrize("Hi", [1, 4, 8, 12, 16])
def test_fp8_heads(Hi):
    spec = spec_by_name("b8_ctx64k").replace(batch=2, seq_len=(20000, 9), heads=8, idx_heads=Hi, topk=300)
    w = Workload(spec)
    idx, sc = _run_indexer(w)
    _check_queries(w, [0, 1], idx, sc)


def test_fp8_di128():
    spec = spec_by_name("b8_ctx64k").replace(batch=1, seq_len=(40000,), heads=8, idx_dim=128)
    w = Workload(spec)
    idx, sc = _run_indexer(w)
    _check_queries(w, [0], idx, sc)


def test_fp8_b8_ctx64k_full():
    w = Workload(spec_by_name("b8_ctx64k").replace(heads=8))
    idx, sc = _run_indexer(w)
    _check_queries(w, range(8), idx, sc)


def test_fp8_needles_in_topk():
    w = Workload(spec_by_name("b1_ctx1m").replace(seq_len=(1 << 18,), heads=8))
    idx, sc = _run_indexer(w)
    assert set(w.needles) <= set(idx[0].tolist())
    _check_queries(w, [0], idx, sc)


def test_prefill_row_mode_causal():
    spec = spec_by_name("prefill_4k_at_128k").replace(seq_len=(8192 + 512,), queries_per_seq=512, heads=8)
    w = Workload(spec)
    idx, sc = _run_indexer(w)
    _check_queries(w, [0, 1, 2, 3, 100, 255, 511], idx, sc)


def test_short_sequences_pad():
    spec = spec_by_name("b8_ctx64k").replace(batch=5, seq_len=(1, 3, 4, 7, 4100), heads=8, topk=1024)
    w = Workload(spec)
    idx, sc = _run_indexer(w)
    assert np.all(idx[0] == -1) and np.all(idx[1] == -1)
    assert idx[2, 0] == 0 and np.all(idx[2, 1:] == -1)
    _check_queries(w, range(5), idx, sc)
