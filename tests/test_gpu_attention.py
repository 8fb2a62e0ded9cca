"""GPU hybrid_decode_attn against the oracle, given the oracle's own top-k
rows (so attention is checked apart from selection): CSA and HCA modes, fp32
and bf16, sink / no sink, short windows, -1 padding, skipped bad indices."""

import numpy as np
import pytest
import torch

from oracle import indexer
from oracle import step as ostep
from synth import Workload, spec_by_name

from compressed_sparse_kv_compress_b200 import api
from helpers import bounds, check_attention, dtypes, np_arrays, to_f64

pytestmark = pytest.mark.gpu


def _oracle_rows(w, a):
    m = w.meta
    rows = np.full((m["T"], m["k"]), -1, np.int64)
    for t in range(m["T"]):
        rows[t] = indexer.topk_select(ostep.query_scores(m, a, dtypes(w), t), m["k"])
    return rows


def _attn(w, dev, mode, idx=None, sink=True, pairs=False):
    m = w.meta
    b = bounds(w)
    T, H = m["T"], m["H"]
    layer = "c" if mode == api.CSA else "h"
    off = dev["csa_off"] if mode == api.CSA else dev["hca_off"]
    ws = api.attn_workspace(mode, T, H, m["k"], m["W"], b["max_hca_visible"])
    out = torch.empty(T, H, 128, dtype=torch.float32, device="cuda")
    lse = torch.empty(T, H, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.hybrid_decode_attn(mode, dev["q_" + layer], dev["cmp_" + layer], off, dev["raw_" + layer], dev["raw_off"],
                           dev["q_seq"], dev["q_pos"], out, ws, window=m["W"], idx=idx, raw_tok0=dev["raw_t0"],
                           sink=dev["sink_" + layer] if sink else None, scale=m["scale"], lse=lse,
                           max_entries=b["max_hca_visible"], adjacent_pairs=pairs, dev_status=st)
    torch.cuda.synchronize()
    return to_f64(out), to_f64(lse), int(st.item())


def _compare(w, dev, a, mode, rows=None, sink=True, extra_rel=None, queries=None, pairs=False):
    m = w.meta
    idx = None if rows is None else torch.from_numpy(rows.astype(np.int32)).cuda()
    o, lse, st = _attn(w, dev, mode, idx, sink, pairs)
    layer = "c" if mode == api.CSA else "h"
    arr = a if sink else {**a, "sink_" + layer: None}
    for t in (queries if queries is not None else range(m["T"])):
        if mode == api.CSA:
            ent = rows[t][(rows[t] >= 0) & (rows[t] < indexer.visible_entries(m["q_pos"][t], 4))]
        else:
            ent = np.arange(indexer.visible_entries(m["q_pos"][t], 128))
        ro, rl, _ = ostep.query_attention(m, arr, dtypes(w), arr["cmp_" + layer], t, layer, ent)
        check_attention(o[t], ro, extra_rel, f"mode {mode} query {t}")
        fin = np.isfinite(rl)
        assert np.allclose(lse[t][fin], rl[fin], rtol=1e-5, atol=1e-5)
    return st


@pytest.mark.parametrize("sink", [True, False])
def test_tiny_fp32_both_modes(sink):
    w = Workload(spec_by_name("tiny").replace(cache="random"))
    a = np_arrays(w)
    dev = w.device("cuda")
    rows = _oracle_rows(w, a)
    assert _compare(w, dev, a, api.CSA, rows, sink, extra_rel=1e-4) == 0
    assert _compare(w, dev, a, api.HCA, None, sink, extra_rel=1e-4) == 0


@pytest.mark.parametrize("H", [8, 64, 128])
def test_bf16_heads(H):
    spec = spec_by_name("b8_ctx64k").replace(batch=3, seq_len=(30001, 2000, 300), heads=H)
    w = Workload(spec)
    a = np_arrays(w)
    dev = w.device("cuda")
    rows = _oracle_rows(w, a)
    assert _compare(w, dev, a, api.CSA, rows) == 0
    assert _compare(w, dev, a, api.HCA) == 0


def test_short_positions_and_padding():
    spec = spec_by_name("b8_ctx64k").replace(batch=4, seq_len=(1, 5, 127, 129), heads=16, topk=64)
    w = Workload(spec)
    a = np_arrays(w)
    dev = w.device("cuda")
    rows = _oracle_rows(w, a)
    assert _compare(w, dev, a, api.CSA, rows) == 0
    assert _compare(w, dev, a, api.HCA) == 0


def test_invisible_index_is_flagged_and_skipped():
    spec = spec_by_name("b8_ctx64k").replace(batch=1, seq_len=(5001,), heads=16, topk=64)
    w = Workload(spec)
    a = np_arrays(w)
    dev = w.device("cuda")
    rows = _oracle_rows(w, a)
    rows[0, 3] = w.meta["ncsa"][0] - 1  # the query's own (incomplete) block: not visible
    rows[0, 5] = -1
    st = _compare(w, dev, a, api.CSA, rows)
    assert st & 1


@pytest.mark.parametrize("Q,sink", [(34, True), (33, True), (8, False)])
def test_hca_adjacent_query_pairs(Q, sink):
    # a prefill-like run of consecutive positions, 64 heads: the HCA kernel takes the queries in
    # pairs (one pass over the union of the two row lists); an odd count leaves the last alone.
    # Positions straddle 128-token block boundaries, so the two queries of a pair can see a
    # different number of entries.
    spec = spec_by_name("prefill_4k_at_128k").replace(seq_len=(20096 + 10,), queries_per_seq=Q, heads=64)
    w = Workload(spec)
    dev = w.device("cuda")
    a = np_arrays(w)
    assert _compare(w, dev, a, api.HCA, sink=sink, pairs=True) == 0
    # and the per-query path agrees to the kernels' rounding (P is rounded to bf16 relative to a
    # running maximum, and the pair's chunks cut the rows elsewhere)
    o1, l1, _ = _attn(w, dev, api.HCA, sink=sink, pairs=True)
    o2, l2, _ = _attn(w, dev, api.HCA, sink=sink, pairs=False)
    assert np.abs(o1 - o2).max() <= 1e-3 * max(1.0, np.abs(o2).max())


def test_hca_pairs_not_adjacent_are_flagged():
    # two sequences of 5 queries: the pair (4, 5) straddles them, which the caller promised not
    # to happen: flagged, and every other query still matches the oracle
    spec = spec_by_name("prefill_4k_at_128k").replace(batch=2, seq_len=(9000, 12000), queries_per_seq=5, heads=64)
    w = Workload(spec)
    dev = w.device("cuda")
    a = np_arrays(w)
    st = _compare(w, dev, a, api.HCA, pairs=True, queries=[0, 1, 2, 3, 4, 6, 7, 8, 9])
    assert st & 1  # CSKV_DEV_BAD_INDEX
