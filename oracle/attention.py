"""Hybrid decode attention: MQA over compressed entries + raw window + sink.

What the pages fix:
* All query heads read one shared set of KV (MQA) ([SW] §十一); grouped
  attention with one group reduces to it ([TR] §2.2, def GQA).
* Logits are QK^T / sqrt(d_k) ([TR] §2.2, def GQA).
* The last 128 tokens keep their raw KV (sliding window) ([SW] §三.1; [AM]);
  the window also covers the tokens of the query's own, not yet complete
  block ([SW] §十); compressed entries and window tokens are concatenated
  before the final attention ([TR] §4.3 改进三).
* CSA attends to the top-k entries the indexer picked ([SW] §六); HCA
  attends densely to every entry ([SW] §八; [TR] §4.3 HCA), with the
  token-granularity window concatenated as well ([TR] §4.3 HCA 拼接).
* An attention sink is an extra position with no content that can absorb
  probability mass, e.g. real KV 0.15, sink 0.85 ([SW] §十二).
* Online softmax with a running max m and sum l equals the full softmax
  exactly ([TR] §3.1).

Readings taken where the pages leave the form open:
* The sink is one logit sigma_h per query head in the softmax denominator
  with a zero value row.
* Window = raw tokens max(0, p-W+1) .. p, the query's own token included;
  no de-duplication against tokens that also sit inside selected entries.
* Rows are packed K||V: K = columns 0..d-1, V = columns d..2d-1.

Parity: pinned (probabilities incl. sink sum to 1, the 0.15 / 0.85 sink
example, MQA == GQA(G=1) via a library attention, dense equivalence for
k >= visible, split-and-merge equals one shot).
"""

from __future__ import annotations

import numpy as np


def attend(q, keys, values, sink=None, scale=1.0):
    """One query's MQA attention with an optional per-head sink logit.

    q [H, d]; keys, values [N, d]; sink [H] or None.  Returns
    (o [H, d], lse [H], p [H, N], p_sink [H]) where p are the probabilities
    of the real rows and p_sink that of the sink (zeros without one).
    """
    q = np.asarray(q, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    values = np.asarray(values, dtype=np.float64)
    H = q.shape[0]
    logits = scale * (q @ keys.T)                                 # [H, N]
    if sink is not None:
        logits = np.concatenate([logits, np.asarray(sink, dtype=np.float64)[:, None]], axis=1)
    if logits.shape[1] == 0:
        return np.zeros((H, values.shape[1])), np.full(H, -np.inf), np.zeros((H, 0)), np.zeros(H)
    m = np.max(logits, axis=1, keepdims=True)
    e = np.exp(logits - m)
    z = np.sum(e, axis=1, keepdims=True)
    p_all = e / z
    n = keys.shape[0]
    p = p_all[:, :n]
    p_sink = p_all[:, n] if sink is not None else np.zeros(H)
    o = p @ values
    lse = (m + np.log(z))[:, 0]
    return o, lse, p, p_sink


def window_tokens(p: int, window: int) -> np.ndarray:
    """Raw token positions the window holds for a query at position p."""
    return np.arange(max(0, int(p) - int(window) + 1), int(p) + 1, dtype=np.int64)


def gather_rows(cmp_rows, entries, raw_rows, raw_tok0, p, window, d):
    """Concatenate the chosen compressed rows and the window's raw rows.

    cmp_rows [Nc, 2d] (decoded), entries: compressed entry indices (>= 0);
    raw_rows [rows, 2d] for tokens raw_tok0, raw_tok0+1, ...
    Returns keys, values [N, d].
    """
    toks = window_tokens(p, window)
    if len(toks) and toks[0] < raw_tok0:
        raise ValueError("window reaches before the provided raw tail")
    ent = np.asarray(entries, dtype=np.int64)
    rows = np.concatenate([np.asarray(cmp_rows)[ent].reshape(len(ent), 2 * d),
                           np.asarray(raw_rows)[toks - raw_tok0].reshape(len(toks), 2 * d)], axis=0)
    return rows[:, :d], rows[:, d:]


def merge_partials(parts, sink=None):
    """Merge split-KV partials, the sink counted once.

    parts: list of (m [H], l [H], acc [H, d]) where, over the split's rows,
    m is the max logit, l = sum exp(logit - m) and acc = sum exp(logit - m) v.
    Returns (o [H, d], lse [H]):
      M = max(max_s m_s, sigma);  L = sum_s e^{m_s-M} l_s + e^{sigma-M}
      o = sum_s e^{m_s-M} acc_s / L;  lse = M + log L.
    """
    ms = np.stack([np.asarray(p[0], dtype=np.float64) for p in parts])   # [S, H]
    ls = np.stack([np.asarray(p[1], dtype=np.float64) for p in parts])
    accs = np.stack([np.asarray(p[2], dtype=np.float64) for p in parts])  # [S, H, d]
    M = np.max(ms, axis=0)
    if sink is not None:
        M = np.maximum(M, np.asarray(sink, dtype=np.float64))
    f = np.exp(ms - M[None, :])
    L = np.sum(f * ls, axis=0)
    if sink is not None:
        L = L + np.exp(np.asarray(sink, dtype=np.float64) - M)
    o = np.sum(f[:, :, None] * accs, axis=0) / L[:, None]
    return o, M + np.log(L)


def partial(q, keys, values, scale=1.0):
    """(m, l, acc) of one split of rows, as merge_partials expects."""
    logits = scale * (np.asarray(q, dtype=np.float64) @ np.asarray(keys, dtype=np.float64).T)
    m = np.max(logits, axis=1)
    e = np.exp(logits - m[:, None])
    return m, np.sum(e, axis=1), e @ np.asarray(values, dtype=np.float64)
