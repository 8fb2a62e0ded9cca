"""Lightning Indexer on MXFP4 vectors (lindex_score_topk_mxfp4) against the oracle: the pages
let the indexer's QK path run in FP4 ([SW] §六.1, §十三.4; [TR] §4.2).  Keys and queries are
E2M1 codes with E8M0 block scales; the oracle decodes them exactly (codecs.mx_fp4_decode) and
scores in float64.  Checked: the scores of the kept entries (fp32 against fp64), and a selection
that may differ from the oracle's only for entries within 1e-4 of the k-th score, in one-query
groups (split mode, a whole grid on one query), several ragged queries at once, and row mode."""

import numpy as np
import pytest
import torch

from compressed_sparse_kv_compress_b200 import api
from oracle import codecs, indexer
from synth import mxfp4_random

from helpers import check_selection

pytestmark = pytest.mark.gpu


def _decode(codes, scales):
    return codecs.mx_fp4_decode(codecs.unpack_nibbles(codes.numpy()), scales.numpy())


def _case(seed, lengths, q_per_seq, Hi, Di, k, scaled_queries=True):
    """Sequences of `lengths` tokens, the last q_per_seq positions of each as queries."""
    B = len(lengths)
    nent = [(n + 3) // 4 for n in lengths]
    ent_off = np.concatenate([[0], np.cumsum(nent)]).astype(np.int64)
    kc, ks = mxfp4_random(seed, "k", int(ent_off[-1]), Di)
    q_seq, q_pos = [], []
    for b, n in enumerate(lengths):
        for j in range(q_per_seq):
            q_seq.append(b)
            q_pos.append(n - q_per_seq + j)
    T = len(q_seq)
    qc, qs = mxfp4_random(seed, "q", T * Hi, Di)
    qc, qs = qc.view(T, Hi, Di // 2), qs.view(T, Hi, Di // 32)
    rng = np.random.default_rng(seed)
    q_scale = torch.from_numpy(rng.uniform(0.5, 2.0, (T, Hi)).astype(np.float32)) if scaled_queries else None
    head_w = torch.from_numpy(rng.uniform(0.25, 1.5, Hi).astype(np.float32))
    return dict(kc=kc, ks=ks, qc=qc, qs=qs, q_scale=q_scale, head_w=head_w, ent_off=ent_off,
                q_seq=np.array(q_seq, np.int32), q_pos=np.array(q_pos, np.int64), k=k, Hi=Hi, Di=Di)


def _run(c):
    d = lambda t: None if t is None else t.cuda()  # noqa: E731
    T = len(c["q_seq"])
    vis = [(p + 1) // 4 for p in c["q_pos"]]
    max_e = max(vis)
    ws = api.lindex_workspace(T, c["k"], max_e)
    idx = torch.full((T, c["k"]), -7, dtype=torch.int32, device="cuda")
    sc = torch.empty(T, c["k"], dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.lindex_score_topk_mxfp4(d(c["qc"]), d(c["qs"]), d(c["kc"]), d(c["ks"]),
                                torch.from_numpy(c["q_seq"]).cuda(), torch.from_numpy(c["q_pos"]).cuda(),
                                torch.from_numpy(c["ent_off"]).cuda(), idx, ws, max_entries=max_e,
                                q_scale=d(c["q_scale"]), head_w=d(c["head_w"]), out_score=sc, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return idx.cpu().numpy(), sc.cpu().numpy()


def _check(c, idx, sc, queries):
    kv = _decode(c["kc"], c["ks"])
    for t in queries:
        b, p = c["q_seq"][t], c["q_pos"][t]
        V = indexer.visible_entries(p, 4)
        e0 = c["ent_off"][b]
        qv = _decode(c["qc"][t], c["qs"][t])
        qsc = None if c["q_scale"] is None else c["q_scale"][t].numpy()
        s = indexer.index_scores(qv, kv[e0:e0 + V], qsc, None, c["head_w"].numpy())
        check_selection(idx[t], s, c["k"], f"query {t}")
        kk = min(c["k"], V)
        sel = idx[t, :kk]
        err = np.abs(sc[t, :kk] - s[sel])
        assert err.max(initial=0) <= 1e-5 * max(1.0, np.abs(s).max(initial=0)), f"query {t}: score error"


@pytest.mark.parametrize("Hi,Di", [(8, 64), (16, 64), (8, 128), (4, 128), (12, 64)])
def test_one_query_split_mode(Hi, Di):
    c = _case(Hi * 1000 + Di, [1 << 18], 1, Hi, Di, 1024)
    idx, sc = _run(c)
    _check(c, idx, sc, [0])


def test_ragged_queries_split_mode():
    c = _case(7, [65536, 40001, 9000, 300, 4, 1], 1, 8, 64, 1024, scaled_queries=False)
    idx, sc = _run(c)
    assert np.all(idx[5] == -1) and idx[4, 0] == 0 and np.all(idx[4, 1:] == -1)
    _check(c, idx, sc, range(6))


def test_many_queries_row_mode():
    # 512 queries of one sequence (a prefill chunk): the CTAs own whole queries
    c = _case(9, [8192 + 512], 512, 8, 64, 512)
    idx, sc = _run(c)
    _check(c, idx, sc, [0, 1, 255, 511])


def test_unit_codes_give_exact_integer_scores():
    # every element code 0x2 (1.0) and scale 2^0: each head's dot product is Di exactly, and the
    # scores are equal, so the selection is the lowest indices (ties to the lower index)
    Di, Hi, V = 64, 8, 5000
    c = _case(11, [4 * V], 1, Hi, Di, 100, scaled_queries=False)
    c["kc"][:] = 0x22
    c["ks"][:] = 127
    c["qc"][:] = 0x22
    c["qs"][:] = 127
    c["head_w"][:] = 1.0
    idx, sc = _run(c)
    assert np.array_equal(idx[0], np.arange(100))
    assert np.all(sc[0] == Hi * Di)
