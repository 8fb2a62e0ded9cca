"""End-to-end GPU decode step (compress -> index/top-k -> CSA and HCA attention)
against the oracle's step on the same seeded inputs, at small sizes and at the
full workload sizes (sampled queries), eager, two-stream and graph-replayed."""

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import indexer
from oracle import step as ostep
from synth import Workload, spec_by_name

from helpers import bulk_bounds, check_attention, check_selection, compress_tol_check, decode_step, dtypes, \
    np_arrays, storage_rows, to_f64

pytestmark = pytest.mark.gpu


def _run_gpu(w, two_streams=False, graph=False):
    step, dev = decode_step(w, two_streams=two_streams)
    if w.spec.cache == "compress":
        step.bulk_compress(*bulk_bounds(w))
    if graph:
        step.capture()
        step.replay()
    else:
        step.run()
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0, f"device status {int(step.status.item())}"
    return step, dev


def _check(w, step, dev, queries, extra_rel=None):
    m, a = w.meta, np_arrays(w)
    res = ostep.run_step(m, a, dtypes(w), queries=queries, bulk=(w.spec.cache == "compress"))
    # caches: the step's recompressed entries
    for b in range(m["B"]):
        for layer, key, off in (("csa", "cmp_c", "csa_off"), ("hca", "cmp_h", "hca_off")):
            ents, ref = res["new"][(layer, b)]
            got = storage_rows(dev[key][m[off][b] + ents[0]: m[off][b] + ents[-1] + 1])
            compress_tol_check(got, ref, w.spec.dtype, f"{layer} seq{b}")
    idx = step.idx.cpu().numpy()
    o_c, o_h = to_f64(step.o_c), to_f64(step.o_h)
    lse_c = to_f64(step.lse_c)
    arrays_after = {**a, "cmp_c": res["cmp_c"], "cmp_h": res["cmp_h"]}
    n_diff = 0
    for j, t in enumerate(queries):
        n_diff += check_selection(idx[t], res["scores"][j], m["k"], f"query {t}")
        sel = idx[t][idx[t] >= 0]
        if np.array_equal(sel, res["idx"][j][res["idx"][j] >= 0]):
            ref_c = res["o_c"][j]
            np.testing.assert_allclose(lse_c[t], res["lse_c"][j], rtol=1e-5, atol=1e-5)
        else:  # an allowed near-tie swap: attend over the GPU's selection
            ref_c = ostep.query_attention(m, arrays_after, dtypes(w), res["cmp_c"], t, "c", sel)[0]
        check_attention(o_c[t], ref_c, extra_rel, f"CSA query {t}")
        check_attention(o_h[t], res["o_h"][j], extra_rel, f"HCA query {t}")
    return res, n_diff


@pytest.mark.parametrize("name", ["tiny", "tiny_bias"])
def test_tiny_fp32(name):
    w = Workload(spec_by_name(name))
    step, dev = _run_gpu(w)
    _check(w, step, dev, [0], extra_rel=1e-4)


def test_small_bf16_two_streams_graph_equal_eager():
    spec = spec_by_name("ragged_b64").replace(batch=6, len_range=(3000, 40000), heads=64)
    w = Workload(spec)
    s1, d1 = _run_gpu(w)
    _check(w, s1, d1, list(range(6)))
    w2 = Workload(spec)
    s2, _ = _run_gpu(w2, two_streams=True, graph=True)
    assert torch.equal(s1.idx, s2.idx)
    assert torch.equal(s1.o_c, s2.o_c) and torch.equal(s1.o_h, s2.o_h)


@pytest.mark.parametrize("zero_copy", [True, False, None])
def test_graph_with_host_copies_equals_eager(zero_copy):
    # capture_io: new queries copied from pinned host memory and both outputs read back, all
    # inside the step's graph (zero copy: the kernels read and write the host buffers over the
    # bus; otherwise through copies); replayed twice with different queries
    spec = spec_by_name("ragged_b64").replace(batch=3, len_range=(3000, 20000), heads=64)
    w = Workload(spec)
    step, dev = decode_step(w, two_streams=True)
    qs = [dev["q_c"].clone(), dev["q_c"].flip(1).contiguous()]  # two query sets (heads reversed)
    h_q = torch.empty(dev["q_c"].shape, dtype=dev["q_c"].dtype, pin_memory=True)
    h_oc = torch.empty(step.o_c.shape, dtype=step.o_c.dtype, pin_memory=True)
    h_oh = torch.empty(step.o_h.shape, dtype=step.o_h.dtype, pin_memory=True)
    views = step.capture_io([(h_q, dev["q_c"])], [(step.o_c, h_oc), (step.o_h, h_oh)], zero_copy=zero_copy)
    for q in qs:
        views[0].copy_(q.cpu())
        step.replay_io()
        torch.cuda.synchronize()
        assert int(step.status.item()) == 0
        got_c, got_h = h_oc.clone(), h_oh.clone()
        dev["q_c"].copy_(q)
        step.run()
        torch.cuda.synchronize()
        assert torch.equal(got_c, step.o_c.cpu()) and torch.equal(got_h, step.o_h.cpu())


def test_b8_ctx64k_full():
    w = Workload(spec_by_name("b8_ctx64k"))
    step, dev = _run_gpu(w, two_streams=True)
    _check(w, step, dev, list(range(8)))


def test_b1_ctx1m_full_with_needles():
    w = Workload(spec_by_name("b1_ctx1m"))
    step, dev = _run_gpu(w, two_streams=True, graph=True)
    assert set(w.needles) <= set(step.idx[0].cpu().tolist())
    _check(w, step, dev, [0])


def test_ragged_b64_full_sampled():
    w = Workload(spec_by_name("ragged_b64"))
    step, dev = _run_gpu(w, two_streams=True)
    n = w.meta["n"]
    queries = sorted({0, 63, int(np.argmax(n)), int(np.argmin(n)), 17, 40})
    _check(w, step, dev, queries)


def test_prefill_chunk_full_sampled():
    # 4096 queries: the indexer takes its tensor-core path (16-query tiles) and the attention its
    # many-query plan; the first and last query of every 128-query block, and a few between
    w = Workload(spec_by_name("prefill_4k_at_128k"))
    step, dev = _run_gpu(w)
    T = w.meta["T"]
    queries = sorted({q for b in range(0, T, 128) for q in (b, b + 127)} | {1, 2, 3, 15, 16, 1001, 2048, 4094})
    assert len(queries) >= 64
    _check(w, step, dev, queries)


def _issue_layers(step, order):
    main = torch.cuda.current_stream()
    step.side.wait_stream(main)
    if order == "csa_first":
        step.csa_layer(main)
        step.hca_layer(step.side)
    else:
        step.hca_layer(step.side)
        step.csa_layer(main)
    main.wait_stream(step.side)


@pytest.mark.parametrize("name,reps", [("ragged_b64", 20), ("b8_ctx64k", 12), ("b1_ctx1m", 12)])
def test_selection_stable_beside_hca_layer(name, reps):
    # The HCA layer's kernels share the SMs with the indexer when it runs on a second stream,
    # issued before or after the CSA layer.  Every repetition, in both issue orders and as a
    # replayed two-stream graph, must select exactly what a one-stream run selects (the
    # selection is deterministic), and that run must match the oracle on sampled queries.
    w = Workload(spec_by_name(name))
    m, a = w.meta, np_arrays(w)
    step, dev = decode_step(w)
    step.run()
    torch.cuda.synchronize()
    ref = step.idx.clone()
    T = m["T"]
    for t in sorted({0, T // 2, T - 1}):
        check_selection(ref[t].cpu().numpy(), ostep.query_scores(m, a, dtypes(w), t), m["k"], f"query {t}")
    step2, _ = decode_step(w, dev=dev, two_streams=True)
    for order in ("csa_first", "hca_first"):
        for rep in range(reps):
            step2.idx.fill_(-2)
            _issue_layers(step2, order)
            torch.cuda.synchronize()
            assert int(step2.status.item()) == 0
            bad = (step2.idx != ref).any(dim=1).nonzero().flatten().tolist()
            assert not bad, f"{order} repetition {rep}: queries {bad} select differently"
    step2.capture()
    for rep in range(reps):
        step2.idx.fill_(-2)
        step2.replay()
        torch.cuda.synchronize()
        assert int(step2.status.item()) == 0
        assert torch.equal(step2.idx, ref), f"graph replay {rep} selects differently"


def test_step_pools_its_entries_keys():
    # per-token indexer keys: the CSA compression of the step also pools its entries' keys
    # (fused), the indexer reads them; the codes are checked against the exact fp64 pooling
    # (band rule) and the selection and outputs against the oracle's step with pooled keys
    from helpers import check_pooled_keys
    spec = spec_by_name("b8_ctx64k").replace(batch=4, seq_len=(65536, 30001, 4097, 4100), heads=64, pool_keys=True)
    w = Workload(spec)
    step, dev = _run_gpu(w, two_streams=True)
    m, a = w.meta, np_arrays(w)
    codes, scales = dev["k_idx"].cpu().numpy(), dev["k_scale"].cpu().numpy()
    for b in range(m["B"]):
        ents, _, _ = ostep.pooled_step_keys(m, a, b)
        o = m["csa_x_off"][b]
        tok = storage_rows(w.arrays["k_tok"][o + 4 * ents[0] - m["csa_t0"][b]: o + m["n"][b] - m["csa_t0"][b]])
        rows = m["csa_off"][b] + ents
        check_pooled_keys(codes[rows], scales[rows], tok, 4, what=f"seq {b}")
    _check(w, step, dev, list(range(m["T"])))
