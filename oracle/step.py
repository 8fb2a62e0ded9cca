"""One decode (or prefill-chunk) step of the hybrid path, end to end, in fp64.

The step, per sequence and per query, in the order the pages give it:
1. compress the CSA and HCA entries that contain the step's new tokens
   (or every entry, when building a cache from scratch) and store them in
   the cache's storage format;
2. score every visible CSA entry with the Lightning Indexer and keep the
   top-k;
3. CSA attention over the top-k entries + the raw window + the sink;
4. HCA attention over every visible HCA entry + the raw window + the sink.
([SW] §三-§十二; [TR] §4.2-§4.3.)

Inputs are storage-form numpy arrays keyed by name, and plain ints/lists in
``meta``; the key names are the ones the synthetic workloads use:
  caches   cmp_c [sum ceil(n/4), 2d], cmp_h [sum ceil(n/128), 2d]
  rows     x_a z_a x_b z_b (tail from csa_t0[b]), x_h z_h (from hca_t0[b]),
           raw_c raw_h (from raw_t0[b]); row offsets csa_x_off, hca_x_off, raw_off
  indexer  k_idx [sum ceil(n/4), di] (+ k_scale), q_idx [T, Hi, di] (+ q_scale), head_w
  queries  q_c q_h [T, H, d], sink_c sink_h [H], q_seq [T], q_pos [T]
  biases   bias_a bias_b [4, 2d], bias_h [128, 2d] (or None)
``dtypes`` gives the storage formats: {'kv': 'bf16'|'f32', 'idx': 'fp8'|'f32'}.
"""

from __future__ import annotations

import numpy as np

from . import attention, codecs, compress, indexer


def _rows(arrays, name, dt, off, r0, r1):
    a = arrays[name]
    return codecs.decode(a[off + r0: off + r1], dt)


def compress_step(meta, arrays, dtypes, bulk=False, seqs=None):
    """Compress the step's entries into copies of both caches.

    Returns (cmp_c, cmp_h, new) where the caches are storage-form copies with
    the recomputed entries written, and ``new[(layer, b)] = (entries, f64 rows)``.
    """
    kv = dtypes["kv"]
    cmp_c = arrays["cmp_c"].copy()
    cmp_h = arrays["cmp_h"].copy()
    new = {}
    bias = {k: (None if arrays.get(k) is None else np.asarray(arrays[k], dtype=np.float64))
            for k in ("bias_a", "bias_b", "bias_h")}
    for b in (range(meta["B"]) if seqs is None else seqs):
        n = meta["n"][b]
        # CSA layer: two streams over the tail rows starting at token csa_t0[b].
        first = 0 if bulk else meta["csa_first"][b]
        num = meta["ncsa"][b] if bulk else meta["csa_num"][b]
        ents = np.arange(first, first + num)
        o, r = meta["csa_x_off"][b], meta["csa_x_off"][b + 1] - meta["csa_x_off"][b]
        xa, za, xb, zb = (_rows(arrays, nm, kv, o, 0, r) for nm in ("x_a", "z_a", "x_b", "z_b"))
        rows = compress.csa_compress(ents, n, xa, za, xb, zb, bias["bias_a"], bias["bias_b"],
                                     tok0=meta["csa_t0"][b])
        cmp_c[meta["csa_off"][b] + ents] = codecs.encode(rows, kv)
        new[("csa", b)] = (ents, rows)
        # HCA layer: one stream over the tail rows starting at token hca_t0[b].
        first = 0 if bulk else meta["hca_first"][b]
        num = meta["nhca"][b] if bulk else meta["hca_num"][b]
        ents = np.arange(first, first + num)
        o, r = meta["hca_x_off"][b], meta["hca_x_off"][b + 1] - meta["hca_x_off"][b]
        xh, zh = (_rows(arrays, nm, kv, o, 0, r) for nm in ("x_h", "z_h"))
        rows = compress.hca_compress(ents, n, xh, zh, bias["bias_h"], tok0=meta["hca_t0"][b])
        cmp_h[meta["hca_off"][b] + ents] = codecs.encode(rows, kv)
        new[("hca", b)] = (ents, rows)
    return cmp_c, cmp_h, new


def pooled_step_keys(meta, arrays, b):
    """With per-token indexer keys (``k_tok``, rows indexed like x_a): the step's CSA entries of
    sequence b get keys pooled from their tokens ([TR] §4.2; the exact definition,
    indexer.pool_keys_f64 / quantize_keys_f64).  Returns (entries, E4M3 codes, scales)."""
    first, num = meta["csa_first"][b], meta["csa_num"][b]
    ents = np.arange(first, first + num)
    t0, n = meta["csa_t0"][b], meta["n"][b]
    o = meta["csa_x_off"][b]
    tok = codecs.decode(arrays["k_tok"][o + 4 * first - t0: o + n - t0], "bf16")
    codes, scales = indexer.quantize_keys_f64(indexer.pool_keys_f64(tok, compress.CSA_RATIO))
    return ents, codes, scales


def query_scores(meta, arrays, dtypes, t):
    """Indexer scores [V] of query t over its visible CSA entries (with ``k_tok``: the step's
    entries scored with their pooled keys)."""
    b, p = meta["q_seq"][t], meta["q_pos"][t]
    V = min(indexer.visible_entries(p, compress.CSA_RATIO), meta["ncsa"][b])
    off = meta["csa_off"][b]
    k_idx = codecs.decode(arrays["k_idx"][off: off + V], dtypes["idx"])
    k_scale = None if arrays.get("k_scale") is None else np.array(arrays["k_scale"][off: off + V], dtype=np.float64)
    if arrays.get("k_tok") is not None:
        ents, codes, scales = pooled_step_keys(meta, arrays, b)
        keep = ents < V
        k_idx[ents[keep]] = codecs.e4m3_decode(codes[keep])
        k_scale[ents[keep]] = scales[keep]
    q_idx = codecs.decode(arrays["q_idx"][t], dtypes["idx"])
    q_scale = None if arrays.get("q_scale") is None else arrays["q_scale"][t]
    return indexer.index_scores(q_idx, k_idx, q_scale, k_scale, arrays.get("head_w"))


def query_attention(meta, arrays, dtypes, cmp, t, layer, entries, cmp_decoded=False):
    """(o [H, d], lse [H], p_sink [H]) of query t in layer 'c' (CSA) or 'h' (HCA).
    cmp_decoded: `cmp` already holds float64 values (e.g. FP8 main-KV rows decoded by
    kv8.decode_rows) instead of rows in the workload's storage dtype."""
    kv, d = dtypes["kv"], meta["d"]
    b, p = meta["q_seq"][t], meta["q_pos"][t]
    off = meta["csa_off"][b] if layer == "c" else meta["hca_off"][b]
    ent = np.asarray(entries, dtype=np.int64)
    if not len(ent):
        cmp_rows = np.zeros((0, 2 * d))
    elif cmp_decoded:
        cmp_rows = np.asarray(cmp[off + ent], dtype=np.float64)
    else:
        cmp_rows = codecs.decode(cmp[off + ent], kv)
    ro, r1 = meta["raw_off"][b], meta["raw_off"][b + 1]
    raw = codecs.decode(arrays["raw_" + layer][ro:r1], kv)
    keys, values = attention.gather_rows(cmp_rows, np.arange(len(ent)), raw, meta["raw_t0"][b], p,
                                         meta["W"], d)
    q = codecs.decode(arrays["q_" + layer][t], kv)
    sink = arrays.get("sink_" + layer)
    o, lse, _, p_sink = attention.attend(q, keys, values, sink, meta["scale"])
    return o, lse, p_sink


def run_step(meta, arrays, dtypes, queries=None, bulk=False):
    """The whole step for the listed queries (all when None).

    Returns a dict: caches after compression ('cmp_c', 'cmp_h', 'new'), and per
    listed query: 'scores' (list of [V]), 'idx' [Tq, k], 'kth' [Tq],
    'o_c', 'lse_c', 'psink_c', 'o_h', 'lse_h', 'psink_h'.
    """
    queries = list(range(meta["T"])) if queries is None else list(queries)
    cmp_c, cmp_h, new = compress_step(meta, arrays, dtypes, bulk=bulk)
    H, d, k = meta["H"], meta["d"], meta["k"]
    res = dict(cmp_c=cmp_c, cmp_h=cmp_h, new=new, queries=queries, scores=[],
               idx=np.full((len(queries), k), -1, dtype=np.int64), kth=np.zeros(len(queries)))
    for name in ("o_c", "o_h"):
        res[name] = np.zeros((len(queries), H, d))
    for name in ("lse_c", "lse_h", "psink_c", "psink_h"):
        res[name] = np.zeros((len(queries), H))
    for j, t in enumerate(queries):
        s = query_scores(meta, arrays, dtypes, t)
        sel = indexer.topk_select(s, k)
        res["scores"].append(s)
        res["idx"][j] = sel
        res["kth"][j] = indexer.kth_score(s, k)
        res["o_c"][j], res["lse_c"][j], res["psink_c"][j] = query_attention(
            meta, arrays, dtypes, cmp_c, t, "c", sel[sel >= 0])
        b, p = meta["q_seq"][t], meta["q_pos"][t]
        vh = min(indexer.visible_entries(p, compress.HCA_RATIO), meta["nhca"][b])
        res["o_h"][j], res["lse_h"][j], res["psink_h"][j] = query_attention(
            meta, arrays, dtypes, cmp_h, t, "h", np.arange(vh))
    return res
