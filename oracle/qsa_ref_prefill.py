"""Plain CPU oracle of QSA sparse prefill (many query tokens per request,
each with its own selection).

TEST INFRASTRUCTURE ONLY, under the same rules as ``qsa_ref``: only
``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may
import it, and it shares no code with the CUDA library.

What the pages say: the blog page ("Qwen 4 QSA 迎来解码上下文并行…", section
"为什么一篇关于未发布架构的 serving PR 仍然值得你花时间") names a separate native
sparse-prefill kernel for the QSA path (PR #59010) and nothing about what it
computes.  The reading used here is the plainest one the decode path
supports: prefill token p is a causal query over its prefix [0, p], and is
computed exactly like a decode query at that position:

* compressed keys as seen at p: blocks 0 .. floor(p/4), the block holding p
  summing only its tokens <= p (the caches are updated before selection, and
  a token does not see later ones);
* scores of those floor(p/4) + 1 blocks against token p's own indexer query,
  top-k selection as in the decode path (higher score first, lower block
  index on ties; ascending; -1 padded);
* exact softmax attention of token p's query over the selected blocks'
  tokens up to p (``qsa_ref.token_set`` with L = p + 1, T = 1).

So a token of the first 2,048 positions (at most 512 blocks) keeps every
block and attends densely and causally.

Pins: ``tests/test_oracle_prefill.py`` (a hand-worked example in
``tests/golden/prefill_hand.json``, dense causal attention from scipy for
p < 2048, a brute-force selection with explicit loops, equality of the last
token with the decode oracle, and causality).
"""
from __future__ import annotations

import numpy as np

from oracle import qsa_ref as ref


def prefix_block_keys(k_idx: np.ndarray, p: int) -> np.ndarray:
    """Compressed keys of blocks 0 .. floor(p/4) as token p sees them: the
    integer sums of the raw keys of tokens <= p.  int64 [p//4 + 1, d]."""
    return ref.compress_keys(np.asarray(k_idx)[: p + 1])


def prefill_token(k_idx: np.ndarray, q_idx_p: np.ndarray, q_p: np.ndarray, K, V, p: int,
                  topk: int, sm_scale: float) -> dict:
    """Token p of a prefill: scores, selection row, o [Hq, D], lse [Hq]."""
    kc = prefix_block_keys(k_idx, p)
    scores = ref.block_scores(q_idx_p, kc)
    sel = ref.select_blocks(scores, topk)
    toks = ref.token_set(sel, p + 1, 1, 0)
    o, lse = ref.attention(q_p, K, V, toks, sm_scale)
    return dict(scores=scores, sel=sel, o=o, lse=lse)


def prefill_request(k_idx: np.ndarray, q_idx: np.ndarray, q: np.ndarray, K, V, p_first: int,
                    topk: int, sm_scale: float) -> dict:
    """Query tokens p_first .. L-1 of one request (L = k_idx rows).

    k_idx int8 [L, d] raw indexer keys; q_idx int8 [L - p_first, d] the
    query tokens' indexer queries; q float64 [L - p_first, Hq, D]; K, V
    float64 [L, Hkv, D] (or StoredRows).  Returns per-token lists of scores
    and arrays sel [n, topk], o [n, Hq, D], lse [n, Hq]."""
    L = np.asarray(k_idx).shape[0]
    out = [prefill_token(k_idx, q_idx[i], q[i], K, V, p, topk, sm_scale)
           for i, p in enumerate(range(p_first, L))]
    return dict(scores=[x["scores"] for x in out],
                sel=np.stack([x["sel"] for x in out]) if out else np.zeros((0, topk), np.int32),
                o=np.stack([x["o"] for x in out]) if out else None,
                lse=np.stack([x["lse"] for x in out]) if out else None)
