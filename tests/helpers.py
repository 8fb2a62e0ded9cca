"""Glue shared by the GPU parity tests: synthetic workload -> CUDA library
calls on one side, -> oracle on the other, and the comparison rules."""

from __future__ import annotations

import numpy as np
import torch

from oracle import codecs, indexer
from synth import Workload

# Parity tolerances of the hot path (bf16 in, fp32 accumulate, against the fp64 oracle):
ATTN_MAX_REL = 1e-2      # attention outputs: max|d| <= 1e-2 * max|ref|
ATTN_MEAN_ABS = 1e-3     # attention outputs: mean|d| <= 1e-3
SEL_BAND = 1e-4          # end-to-end top-k may differ only for entries within 1e-4 of the k-th score


def np_arrays(w: Workload) -> dict:
    return {k: w.numpy(k) for k in w.arrays}


def dtypes(w: Workload) -> dict:
    return {"kv": w.spec.dtype, "idx": w.spec.idx_dtype}


def bounds(w: Workload) -> dict:
    m = w.meta
    return dict(
        max_csa_blocks=max(m["csa_num"]), max_hca_blocks=max(m["hca_num"]),
        max_csa_visible=max(indexer.visible_entries(p, 4) for p in m["q_pos"]),
        max_hca_visible=max(indexer.visible_entries(p, 128) for p in m["q_pos"]),
    )


def adjacent_pairs(w: Workload) -> bool:
    """Queries 2j, 2j + 1 are one sequence's consecutive positions (every sequence has an even
    number of queries, at its last positions)."""
    Q = w.meta["Q"]
    return Q >= 2 and Q % 2 == 0


def decode_step(w: Workload, dev=None, two_streams=False):
    from compressed_sparse_kv_compress_b200 import DecodeStep
    dev = dev if dev is not None else w.device("cuda")
    m = w.meta
    step = DecodeStep(dev, k=m["k"], window=m["W"], scale=m["scale"], two_streams=two_streams,
                      adjacent_pairs=adjacent_pairs(w), **bounds(w))
    return step, dev


def bulk_bounds(w: Workload):
    return max(w.meta["ncsa"]), max(w.meta["nhca"])


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def check_attention(o_gpu, o_ref, extra_rel=None, what=""):
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    d = np.abs(o_gpu - o_ref)
    mx = np.abs(o_ref).max()
    assert d.max() <= ATTN_MAX_REL * mx, f"{what}: max|d| {d.max():.3e} > {ATTN_MAX_REL} * {mx:.3e}"
    assert d.mean() <= ATTN_MEAN_ABS, f"{what}: mean|d| {d.mean():.3e}"
    if extra_rel is not None:
        assert d.max() <= extra_rel * mx, f"{what}: max|d| {d.max():.3e} > {extra_rel} * {mx:.3e}"
    return d.max() / max(mx, 1e-300)


def check_selection(gpu_row, scores, k, what=""):
    """gpu_row: int row [k] (ascending, -1 padded); scores: oracle float64 scores [V]."""
    gpu_row = np.asarray(gpu_row, dtype=np.int64)
    V = len(scores)
    kk = min(k, V)
    ref = indexer.topk_select(scores, k)
    assert np.all(gpu_row[kk:] == -1), f"{what}: padding"
    sel = gpu_row[:kk]
    assert np.all(np.diff(sel) > 0), f"{what}: not strictly ascending"
    assert sel.min(initial=0) >= 0 and sel.max(initial=-1) < V, f"{what}: out of range"
    diff = np.setxor1d(sel, ref[:kk])
    if len(diff):
        sk = indexer.kth_score(scores, k)
        far = diff[np.abs(scores[diff] - sk) > SEL_BAND]
        assert len(far) == 0, f"{what}: {len(far)} entries differ outside the 1e-4 band, e.g. {far[:5]}"
    return len(diff)


def compress_tol_check(gpu_rows, ref64, dtype, what=""):
    gpu_rows = np.asarray(gpu_rows, dtype=np.float64)
    mx = np.abs(ref64).max()
    d = np.abs(gpu_rows - ref64)
    if dtype == "bf16":
        bound = 2.0 ** -8 * np.abs(ref64) + 1e-6 * mx
    else:
        bound = 1e-5 * mx + 0 * ref64
    bad = d > bound
    assert not bad.any(), f"{what}: {bad.sum()} elements off, worst {d.max():.3e} (max|ref| {mx:.3e})"
    return d.max()


def storage_rows(t: torch.Tensor) -> np.ndarray:
    """Device cache rows -> float64 via the oracle's codecs (bf16 decoded exactly)."""
    c = t.detach().cpu()
    if c.dtype == torch.bfloat16:
        return codecs.bf16_decode(c.view(torch.int16).numpy().view(np.uint16))
    return c.numpy().astype(np.float64)


def check_pooled_keys(gpu_codes, gpu_scale, tok_f64, ratio=4, what=""):
    """Pooled indexer keys from the GPU against the exact (fp64) definition.

    Outside the fp32 error band (oracle.indexer.quotient_error_bound) every code must equal
    the exact code; inside it, the decoded value must lie between the codes of the band's
    two ends (the neighbouring code is as correct as the exact one there).  Scales must lie
    within their bound.  Returns the number of elements inside the band."""
    key = indexer.pool_keys_f64(tok_f64, ratio)
    c64, s64 = indexer.quantize_keys_f64(key)
    tol_v, tol_s = indexer.quotient_error_bound(tok_f64, ratio)
    v64 = key / s64[:, None]
    lo = codecs.e4m3_decode(codecs.e4m3_encode(v64 - tol_v))
    hi = codecs.e4m3_decode(codecs.e4m3_encode(v64 + tol_v))
    got = codecs.e4m3_decode(np.asarray(gpu_codes, dtype=np.uint8))
    sure = lo == hi
    off = sure & (got != codecs.e4m3_decode(c64))
    assert not off.any(), f"{what}: {int(off.sum())} codes differ from the exact ones outside the band"
    out = ~((got >= lo) & (got <= hi))
    assert not out.any(), f"{what}: {int(out.sum())} codes outside the band"
    ds = np.abs(np.asarray(gpu_scale, dtype=np.float64) - s64)
    assert np.all(ds <= tol_s), f"{what}: scale off by {ds.max():.3e}"
    return int((~sure).sum())
