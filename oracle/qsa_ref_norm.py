"""Plain CPU oracle of the normalised-pooling indexer variant (the next
indexer variant after the integer path of ``qsa_ref``).

TEST INFRASTRUCTURE ONLY, under the same rules as ``qsa_ref``: only
``tests/`` may import it, and it shares no code with the CUDA library.

What the pages say ([pr] "PR #53896 完整报告", the ``QSAIndexer.forward``
excerpt under "关键源码片段"): after the indexer's Q/K projection, the token
keys go to the raw-key ring and are pooled by the compress ratio and
normalised before they are written to the compressed-key cache.  The module
list names a Gemma-style RMS norm and a rotary embedding for the indexer
(``apply_qsa_rmsnorm``, ``apply_qsa_rope``).  Neither the kind of pooling nor
that of the normalisation is given.  The reading used here:

* pooling: the mean over the tokens present in the 4-token block (a partial
  tail block averages the tokens it has);
* normalisation: RMS normalisation of the pooled key,
      k_c = p / sqrt(mean_j p_j^2 + eps) * (1 + w),  eps = 1e-6,
  the per-dim weight w entering as (1 + w) as in the Gemma norm (w = 0: none);
* score: q . k_c in float64; selection and output as in the integer path
  (higher score first, then lower block index; ascending, -1 padded).

With floating-point scores a CUDA path and this oracle can order blocks whose
scores differ by rounding differently, so parity is stated by
``selection_within_tolerance``: the kept set must be a top-k of the oracle's
scores up to a tolerance at the threshold.

Pins: ``tests/test_oracle_norm.py`` checks every function against closed
forms, the integer oracle (mean x 4 = sum on full blocks), torch's RMS norm
and brute force.
"""
from __future__ import annotations

import numpy as np

COMPRESS_RATIO = 4
RMS_EPS = 1e-6


def pool_mean(k: np.ndarray) -> np.ndarray:
    """Mean of the raw keys of each 4-token micro-block; a partial tail block
    averages the tokens present.  k: [L, d] -> float64 [ceil(L/4), d]."""
    k = np.asarray(k, dtype=np.float64)
    L, d = k.shape
    n = (L + COMPRESS_RATIO - 1) // COMPRESS_RATIO
    out = np.empty((n, d), dtype=np.float64)
    for b in range(n):
        rows = k[COMPRESS_RATIO * b: min(COMPRESS_RATIO * (b + 1), L)]
        out[b] = rows.sum(axis=0) / rows.shape[0]
    return out


def rms_normalise(x: np.ndarray, eps: float = RMS_EPS, weight: np.ndarray | None = None) -> np.ndarray:
    """RMS normalisation over the last axis, x / sqrt(mean(x^2) + eps), times
    (1 + weight) per dim when a weight is given."""
    x = np.asarray(x, dtype=np.float64)
    y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    if weight is not None:
        y = y * (1.0 + np.asarray(weight, dtype=np.float64))
    return y


def compress_keys_norm(k: np.ndarray, eps: float = RMS_EPS,
                       weight: np.ndarray | None = None) -> np.ndarray:
    """Compressed key of every micro-block: the RMS-normalised mean of its
    tokens' keys.  float64 [ceil(L/4), d]."""
    return rms_normalise(pool_mean(k), eps, weight)


def block_scores_f(q: np.ndarray, kc: np.ndarray, n_sel: int | None = None) -> np.ndarray:
    """Float64 dot product of the indexer query with each compressed key, for
    blocks 0 .. n_sel-1."""
    kc = np.asarray(kc, dtype=np.float64)
    if n_sel is None:
        n_sel = kc.shape[0]
    return kc[:n_sel] @ np.asarray(q, dtype=np.float64)


def select_blocks_f(scores: np.ndarray, topk: int) -> np.ndarray:
    """The topk highest float scores (ties: lower index), ascending, padded
    with -1 to width topk.  int32 [topk]."""
    s = np.asarray(scores, dtype=np.float64)
    n = s.shape[0]
    order = np.lexsort((np.arange(n), -s))
    keep = np.sort(order[: min(topk, n)])
    out = np.full(topk, -1, dtype=np.int32)
    out[: keep.shape[0]] = keep
    return out


def selection_within_tolerance(sel: np.ndarray, scores: np.ndarray, topk: int,
                               atol: float) -> bool:
    """Whether a selection row is an admissible top-k of the oracle's scores:
    ascending, -1 padded, min(topk, n) distinct valid blocks, and with t the
    topk-th largest score, every kept block scores >= t - atol and every
    block left out scores <= t + atol."""
    s = np.asarray(scores, dtype=np.float64)
    n = s.shape[0]
    k = min(topk, n)
    sel = np.asarray(sel)
    kept = sel[sel >= 0]
    if kept.shape[0] != k or np.any(sel[k:] != -1) or np.any(np.diff(kept) <= 0):
        return False
    if k == 0:
        return True
    if kept[-1] >= n:
        return False
    t = np.sort(s)[::-1][k - 1]
    mask = np.zeros(n, dtype=bool)
    mask[kept] = True
    return bool(np.all(s[mask] >= t - atol) and np.all(s[~mask] <= t + atol))
