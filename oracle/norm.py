"""RMSNorm of the queries and of the compressed KV entries (test infrastructure: only the
tests, the smoke check and the bench's CPU baseline use this package).

What the pages fix:
* Among the compensations the design pairs with each loss that compression brings, the
  queries and the KV go through RMSNorm so that attention logits cannot blow up
  ([SW] §十四.3).

Readings taken where the pages leave the form open:
* RMSNorm(x) = x / sqrt(mean_j x_j^2 + eps) * gamma over one 128-dimension head vector:
  every query head, and the K half and the V half of every packed K||V entry row
  separately, each kind with its own gain vector gamma [128] (1 when absent); eps is an
  argument (1e-6 by default).
* The entries are normalised as they are produced (after the compression's weighted sum),
  the queries before the logits.

Parity: pinned (a closed-form example, unit RMS, invariance to a positive scale, sign
equivariance, the gain, a zero vector, the logit bound |<q, k>| <= d that the
normalisation guarantees for unit gains, torch's rms_norm).
"""

from __future__ import annotations

import numpy as np


def rmsnorm(x: np.ndarray, gamma: np.ndarray | None = None, eps: float = 1e-6) -> np.ndarray:
    """RMSNorm over the last axis, in float64."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    y = x / np.sqrt(ms + eps)
    if gamma is not None:
        y = y * np.asarray(gamma, dtype=np.float64)
    return y


def norm_packed_rows(rows: np.ndarray, gamma_k=None, gamma_v=None, eps: float = 1e-6) -> np.ndarray:
    """Packed K||V rows [N, 2d] with the K half and the V half normalised separately."""
    r = np.asarray(rows, dtype=np.float64)
    d = r.shape[-1] // 2
    return np.concatenate([rmsnorm(r[..., :d], gamma_k, eps), rmsnorm(r[..., d:], gamma_v, eps)], axis=-1)
