"""Lightning Indexer scores, causal visibility and exact top-k selection.

What the pages fix:
* The indexer gives every query a cheap relevance score against all
  compressed entries, then only the top-k go on to the main attention
  ([SW] §六 funnel; [TR] §4.2 LightningIndexer: scores = relu(q_idx k_idx^T)).
* Each head's score goes through ReLU before the heads are summed, so one
  strongly positive head is not cancelled by a negative one: heads (8, -7)
  give 8, not 1 ([SW] §七).
* It runs at low precision, FP8 or even FP4 ([SW] §六.1; [TR] §4.2).
* k = 1024 at full scale ([AM]).
* A query reads only compressed blocks that lie strictly before it and are
  complete: token 98 may not read block 24 (tokens 96..99) ([SW] §十).

Readings taken where the pages leave the form open:
* Score of entry i for a query with heads h = 0..Hi-1:
      s_i = sum_h w_h * ReLU(sq_h * sk_i * <q_h, k_i>)
  with per-(query, head) scales sq_h and per-entry scales sk_i of the FP8
  codes (1 when the indexer is stored unscaled) and head weights w_h
  (default 1; the pages sum the heads without weights).
* Entry i (ratio m) is visible to position p iff m*(i+1) <= p+1, i.e. the
  query sees entries 0 .. floor((p+1)/m) - 1.
* Top-k keeps min(k, visible) entries: the largest scores, ties going to the
  lower entry index.  The selected set is returned in ascending index order
  and padded with -1 to length k.

Entry keys from per-token keys ([TR] §4.2: the indexer's keys are projected per
token, then pooled with a 1-D pool whose kernel and stride are the block size, before
the scores): readings taken --
* the pool is the mean over the block's tokens (a partial last block: over the tokens
  it has), block size 4, the CSA ratio;
* the entry key is then stored as E4M3 codes with one fp32 scale per entry,
  scale = amax / 448 (1 when the key is all zeros), code = E4M3(key / scale).

Two forms of the pooling are given.  The definition (``pool_keys_f64`` and
``quantize_keys_f64``) computes the mean, the scale and the quotient exactly in float64
and encodes with the nearest-even E4M3 rule.  The codes are integers decided by floating
point, so an fp32 evaluation (the kernel's precision) may land on the neighbouring code
where the exact quotient lies within the fp32 rounding error of an E4M3 rounding
boundary; ``quotient_error_bound`` bounds that error for any evaluation that sums the
tokens in fp32 and divides in fp32, so a comparison can tell where either code is
correct.  ``pool_keys`` / ``quantize_keys`` take the same steps in fp32 (tokens summed in
order, one division by the count, one division by the scale): a second, labelled
restatement in the kernel's precision, not the definition.

Parity: pinned (worked (8, -7) example, block-24 causal example, brute-force
enumeration of k-subsets on tiny inputs, ties; pooling: integer means, identical tokens,
partial blocks, codes that land on printed E4M3 values, the nearest E4M3 value found by
brute force over every finite code, the fp32 restatement agreeing outside the error band;
the E4M3 codec against the OFP8 values and torch's cast).
"""

from __future__ import annotations

import numpy as np

from oracle import codecs


def visible_entries(p: int, ratio: int) -> int:
    """Number of complete blocks strictly before or ending at position p."""
    return (int(p) + 1) // int(ratio)


def entry_visible(i: int, p: int, ratio: int) -> bool:
    """Entry i (tokens ratio*i .. ratio*i+ratio-1) is complete at position p."""
    return ratio * (int(i) + 1) <= int(p) + 1


def index_scores(q_idx, k_idx, q_scale=None, k_scale=None, head_w=None) -> np.ndarray:
    """Scores [V] of V entries for one query.

    q_idx [Hi, di] and k_idx [V, di] are decoded float64 values; q_scale [Hi],
    k_scale [V] and head_w [Hi] are optional (1 when absent).
    """
    q = np.asarray(q_idx, dtype=np.float64)
    k = np.asarray(k_idx, dtype=np.float64)
    Hi = q.shape[0]
    V = k.shape[0]
    sq = np.ones(Hi) if q_scale is None else np.asarray(q_scale, dtype=np.float64)
    sk = np.ones(V) if k_scale is None else np.asarray(k_scale, dtype=np.float64)
    w = np.ones(Hi) if head_w is None else np.asarray(head_w, dtype=np.float64)
    dots = k @ q.T                                   # [V, Hi]: <q_h, k_i>
    per_head = sq[None, :] * sk[:, None] * dots      # scaled head scores
    return np.sum(w[None, :] * np.maximum(per_head, 0.0), axis=1)


def topk_order(scores: np.ndarray) -> np.ndarray:
    """Entry indices ordered by score descending, ties by index ascending."""
    s = np.asarray(scores, dtype=np.float64)
    return np.lexsort((np.arange(len(s)), -s))


def topk_select(scores: np.ndarray, k: int) -> np.ndarray:
    """The min(k, V) best entries, in ascending index order, padded with -1."""
    order = topk_order(scores)[: min(int(k), len(scores))]
    out = np.full(int(k), -1, dtype=np.int64)
    out[: len(order)] = np.sort(order)
    return out


def kth_score(scores: np.ndarray, k: int) -> float:
    """Score of the last entry that top-k keeps (-inf when nothing is kept)."""
    kk = min(int(k), len(scores))
    if kk == 0:
        return -np.inf
    return float(np.asarray(scores, dtype=np.float64)[topk_order(scores)[kk - 1]])


E4M3_MAX = 448.0


def pool_keys(k_tok: np.ndarray, ratio: int = 4) -> np.ndarray:
    """Per-token keys [n, Di] (values exactly representable in fp32) -> entry keys
    [ceil(n/ratio), Di] float32: the mean of each block's tokens, summed in token order
    in fp32 and divided by the block's token count in fp32."""
    k = np.asarray(k_tok, dtype=np.float32)
    n = k.shape[0]
    out = np.zeros(((n + ratio - 1) // ratio, k.shape[1]), dtype=np.float32)
    for i in range(out.shape[0]):
        rows = k[ratio * i: min(n, ratio * (i + 1))]
        acc = rows[0].copy()
        for r in rows[1:]:
            acc = (acc + r).astype(np.float32)
        out[i] = (acc / np.float32(len(rows))).astype(np.float32)
    return out


def quantize_keys(keys: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Entry keys [V, Di] float32 -> (E4M3 codes [V, Di] uint8, fp32 scales [V]):
    scale = amax / 448 in fp32 (1 for an all-zero key), code = E4M3(key / scale) with the
    division in fp32."""
    k = np.asarray(keys, dtype=np.float32)
    amax = np.max(np.abs(k), axis=1)
    scale = np.where(amax > 0, (amax / np.float32(E4M3_MAX)).astype(np.float32), np.float32(1.0)).astype(np.float32)
    v = (k / scale[:, None]).astype(np.float32)
    return codecs.e4m3_encode(v.astype(np.float64)), scale


def pool_keys_f64(k_tok: np.ndarray, ratio: int = 4) -> np.ndarray:
    """Per-token keys [n, Di] -> entry keys [ceil(n/ratio), Di] float64: the exact mean of
    each block's tokens (a partial last block: of the tokens it has)."""
    k = np.asarray(k_tok, dtype=np.float64)
    n = k.shape[0]
    out = np.zeros(((n + ratio - 1) // ratio, k.shape[1]), dtype=np.float64)
    for i in range(out.shape[0]):
        out[i] = np.mean(k[ratio * i: min(n, ratio * (i + 1))], axis=0)
    return out


def quantize_keys_f64(keys: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Entry keys [V, Di] float64 -> (E4M3 codes [V, Di] uint8, scales [V] float64):
    scale = amax / 448 (1 for an all-zero key), code = E4M3(key / scale), every step exact
    in float64 before the one rounding of the encoder."""
    k = np.asarray(keys, dtype=np.float64)
    amax = np.max(np.abs(k), axis=1)
    scale = np.where(amax > 0, amax / E4M3_MAX, 1.0)
    return codecs.e4m3_encode(k / scale[:, None]), scale


def quotient_error_bound(k_tok: np.ndarray, ratio: int = 4) -> tuple[np.ndarray, np.ndarray]:
    """Bounds on how far an fp32 evaluation of the pooling can land from the exact values:
    (tol_v [V, Di], tol_scale [V]) with |v32 - key/scale| <= tol_v for the quotient the
    encoder rounds and |scale32 - scale| <= tol_scale.

    Error analysis (u = 2^-24, the fp32 unit roundoff): summing c tokens in fp32 in any
    order makes at most c - 1 roundings, each at most u times a partial sum, and every
    partial sum is at most S = sum_c |token_c| in magnitude; the division by c adds u |key|.
    So |key32 - key| <= e = u ((c - 1) S / c + |key|).  The largest magnitude moves by at
    most max_j e_j, so the scale (amax / 448, one more rounding) moves by at most
    d_s = max_j e_j / 448 + u scale, and the quotient key32 / scale32 (one more rounding)
    by at most e / scale + |v| d_s / scale + u |v|, to first order; the bound returned is
    twice that, which covers the second-order terms."""
    k = np.asarray(k_tok, dtype=np.float64)
    n = k.shape[0]
    u = 2.0 ** -24
    V = (n + ratio - 1) // ratio
    key = pool_keys_f64(k, ratio)
    _, scale = quantize_keys_f64(key)
    tol_v = np.zeros_like(key)
    tol_s = np.zeros(V)
    for i in range(V):
        rows = k[ratio * i: min(n, ratio * (i + 1))]
        c = rows.shape[0]
        S = np.sum(np.abs(rows), axis=0)
        e = u * ((c - 1) * S / c + np.abs(key[i]))
        ds = np.max(e) / E4M3_MAX + u * scale[i]
        v = np.abs(key[i]) / scale[i]
        tol_v[i] = 2.0 * (e / scale[i] + v * ds / scale[i] + u * v)
        tol_s[i] = 2.0 * ds
    return tol_v, tol_s
