"""Token-dimension compression of KV (CSA 4:1 two-stream, HCA 128:1 one-stream).

What the pages fix:
* CSA turns every 4 consecutive tokens into one compressed KV entry, n -> n/4;
  HCA turns every 128 tokens into one, n -> n/128 ([SW] §二, §三.2-3;
  [AM]; [TR] §4.3 改进一).  10^6 tokens give about 7813 HCA entries
  ([SW] §三.3).
* The entry is a weighted sum of the block's token vectors with learned,
  dynamic weights; averaging is the baseline it improves on; the weights are
  per dimension, not one scalar per token ([SW] §四).
* CSA has two paths: the current block's tokens through path A, the previous
  block's tokens through path B, and both compete together for the
  compression weights ([SW] §五); the two streams carry their own position
  biases B_a, B_b and are normalised by one joint softmax inside the block
  ([TR] §4.3 改进二).  HCA has one stream only ([TR] §4.3, HCA paragraph).

Readings taken where the pages leave the form open:
* "Learned per-dimension weights" = a softmax over the candidate tokens,
  taken separately for every dimension j of the 256-wide packed K||V row:
  w[c, j] = exp(l[c, j]) / sum_c' exp(l[c', j]), C[j] = sum_c w[c, j] x[c, j].
* The logit of a candidate is its per-token, per-dimension logit row plus
  the position bias of its slot inside its block (bias rows are inputs,
  default zero).
* CSA candidates of entry i: tokens 4i..4i+3 through path A (slots 0..3 of
  B_a) and tokens 4(i-1)..4i-1 through path B (slots 0..3 of B_b).  Entry 0
  has no path-B candidates.  A partial last block (n not a multiple of the
  ratio) is compressed over the tokens it has.
* The projections that produce the per-token value and logit rows need
  trained weights and sit outside this path; the rows are inputs.

Parity: pinned (entry counts, mean pooling under uniform logits, one-hot
logits, single-stream reduction, per-dimension independence, overlap reach).
"""

from __future__ import annotations

import numpy as np

CSA_RATIO = 4
HCA_RATIO = 128


def num_entries(n: int, ratio: int) -> int:
    """ceil(n / ratio): a partial last block still yields an entry."""
    return -(-int(n) // int(ratio))


def _softmax_mix(values: np.ndarray, logits: np.ndarray) -> np.ndarray:
    """values, logits [E, C, D] (absent candidates carry logit -inf).

    Per entry and per dimension: softmax over the C candidates, then the
    weighted sum of the candidate values.
    """
    mx = np.max(logits, axis=1, keepdims=True)
    w = np.exp(logits - mx)
    w = w / np.sum(w, axis=1, keepdims=True)
    return np.sum(w * np.where(np.isfinite(logits), values, 0.0), axis=1)


def compress_entries(entries, ratio: int, n: int, cur, prev=None, chunk: int = 2048) -> np.ndarray:
    """Compressed rows (float64, [len(entries), D]) of one sequence of n tokens.

    ``cur`` / ``prev`` are tuples ``(x, z, bias, tok0)``: ``x`` and ``z`` are
    float64 rows [rows, D] for tokens tok0, tok0+1, ...; ``bias`` is None or
    [ratio, D].  ``cur`` supplies the block's own tokens (path A, or the only
    path for HCA); ``prev`` (CSA only) supplies the previous block's tokens
    through path B.
    """
    entries = np.asarray(list(entries), dtype=np.int64)
    x_c, z_c, b_c, t0_c = cur
    D = x_c.shape[1]
    ncand = ratio * (2 if prev is not None else 1)
    out = np.empty((len(entries), D), dtype=np.float64)
    for s in range(0, len(entries), chunk):
        ent = entries[s:s + chunk]
        E = len(ent)
        vals = np.zeros((E, ncand, D))
        logit = np.full((E, ncand, D), -np.inf)
        for slot in range(ratio):
            t = ent * ratio + slot                       # path A / single path: this block
            ok = t < n
            if np.any(ok):
                r = t[ok] - t0_c
                if np.any(r < 0):
                    raise ValueError("token row before the provided tail")
                vals[ok, slot] = x_c[r]
                logit[ok, slot] = z_c[r] + (0.0 if b_c is None else b_c[slot])
        if prev is not None:
            x_p, z_p, b_p, t0_p = prev
            for slot in range(ratio):
                t = (ent - 1) * ratio + slot             # path B: previous block
                ok = ent >= 1
                if np.any(ok):
                    r = t[ok] - t0_p
                    if np.any(r < 0):
                        raise ValueError("token row before the provided tail")
                    vals[ok, ratio + slot] = x_p[r]
                    logit[ok, ratio + slot] = z_p[r] + (0.0 if b_p is None else b_p[slot])
        out[s:s + E] = _softmax_mix(vals, logit)
    return out


def csa_compress(entries, n, x_a, z_a, x_b, z_b, bias_a=None, bias_b=None, tok0=0):
    """CSA entries (two-stream, ratio 4) of one sequence; float64 [E, D]."""
    prev = None if x_b is None else (x_b, z_b, bias_b, tok0)
    return compress_entries(entries, CSA_RATIO, n, (x_a, z_a, bias_a, tok0), prev)


def hca_compress(entries, n, x, z, bias=None, tok0=0):
    """HCA entries (single stream, ratio 128) of one sequence; float64 [E, D]."""
    return compress_entries(entries, HCA_RATIO, n, (x, z, bias, tok0), None, chunk=64)
