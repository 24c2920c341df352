"""Plain CPU oracle for decode-time Qwen Sparse Attention (QSA).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may call it.  It shares no code with the CUDA library.

Everything here is the plain definition of what the method computes, in NumPy,
with exact integers for the indexer and float64 for the attention.  It works
one request at a time on *logical* (de-paged) tensors.

Sources (web pages), cited by title and section:

* [blog]  "Qwen 4 QSA 迎来解码上下文并行：深入解读 vLLM 针对 Qwen3.8-Flash-Next 的草稿 PR"
          (orcarouter.ai), section "拉取请求实际改变了什么": a light indexer
          compresses keys into micro-blocks at ratio 4, scores them, keeps the
          best 512 blocks (about 2,048 token positions); softmax and value
          aggregation run on the uncompressed K/V; under decode context
          parallelism each rank reads its own slice of the KV cache and the
          partial attention results are merged at the end.
* [pr]    "PR #53896 完整报告" (prhub.com.cn), sections "执行摘要" and
          "实现拆解" (weight-free top-k selector over a compressed-key
          cache; MTP step 0 selects and later steps reuse the indices), and
          the ``QSAIndexer.forward`` excerpt under "关键源码片段" (caches are
          updated and compressed before selection; the result is a
          fixed-width, -1-padded, request-relative index row).

Readings where the pages are silent (pooling = plain integer sum, tie-break =
lower block index, output order = ascending block index, partial tail block
competes, softmax scale 1/sqrt(D), split = contiguous slice of logical pages,
MTP token set = selected blocks plus the speculative tail) are those of the
design notes of this repository, each restated at the function that uses it.

Pins: every function below is checked by ``tests/test_oracle.py`` against
closed forms, brute force or library routines, except where a docstring says
"parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

COMPRESS_RATIO = 4  # [blog] "compression ratio 4"; [pr] indexer_compress_ratio
TOPK_BLOCKS = 512   # [blog] "keeps the best 512 blocks"


# ----------------------------------------------------------------------------
# Value decoding (the oracle reads stored bits itself; no GPU conversion)
# ----------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bfloat16 words: the high half of an IEEE-754 binary32."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):                 # NaN payloads stay NaN
        return u32.view(np.float32).astype(np.float64)


def e4m3_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of OCP FP8 E4M3 ("fn": bias 7, no infinities) bytes.

    sign s, exponent e (4 bits), mantissa m (3 bits):
      e == 0            -> (-1)^s * 2^-6 * m/8        (subnormal)
      e == 15 and m == 7 -> NaN
      otherwise          -> (-1)^s * 2^(e-7) * (1 + m/8)
    The FP8 KV cache is an extension beyond the pages (the reference rejects
    FP8 KV for QSA; [pr] "风险与影响").
    """
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    s = (b >> 7) & 1
    e = (b >> 3) & 0xF
    m = b & 0x7
    sign = np.where(s == 1, -1.0, 1.0)
    sub = sign * np.ldexp(m.astype(np.float64) / 8.0, -6)
    nrm = sign * np.ldexp(1.0 + m.astype(np.float64) / 8.0, (e - 7).astype(np.int64))
    out = np.where(e == 0, sub, nrm)
    out = np.where((e == 15) & (m == 7), np.nan, out)
    return out


def decode_values(arr: np.ndarray, kind: str) -> np.ndarray:
    """Stored tensor -> float64.  kind: 'f32' (float32 values), 'bf16'
    (uint16 bit patterns) or 'e4m3' (uint8 bit patterns)."""
    if kind == "f32":
        return np.asarray(arr, dtype=np.float32).astype(np.float64)
    if kind == "bf16":
        return bf16_bits_to_f64(arr)
    if kind == "e4m3":
        return e4m3_bits_to_f64(arr)
    raise ValueError(f"unknown value kind {kind!r}")


class StoredRows:
    """Logical K or V rows [L, Hkv, D] kept as stored (float32 values or
    bf16 / e4m3 bit patterns) with an optional dequantisation scale per
    (token, kv head) [L, Hkv].  Indexing decodes only the rows asked for and
    returns exact float64 values (code * scale for FP8)."""

    def __init__(self, stored: np.ndarray, kind: str, scale: np.ndarray | None = None):
        self.stored, self.kind, self.scale = stored, kind, scale

    @property
    def shape(self):
        return self.stored.shape

    def __getitem__(self, idx):
        vals = decode_values(self.stored[idx], self.kind)
        if self.scale is None:
            return vals
        idx = idx if isinstance(idx, tuple) else (idx,)
        sc = self.scale[idx[:2]].astype(np.float64)
        return vals * sc[..., None] if vals.ndim > sc.ndim else vals * sc


# ----------------------------------------------------------------------------
# Indexer: compression, scoring, selection
# ----------------------------------------------------------------------------

def num_blocks(L: int) -> int:
    """Micro-blocks covering L tokens: ceil(L / 4).  A partial tail block
    exists and competes ([blog] micro-blocks at ratio 4; tail reading)."""
    return (int(L) + COMPRESS_RATIO - 1) // COMPRESS_RATIO


def compress_keys(k_idx: np.ndarray) -> np.ndarray:
    """Compressed key of every micro-block: the integer sum of the (up to) 4
    raw indexer keys it covers.

    k_idx: int8 [L, d] raw indexer keys in logical token order.
    returns int64 [ceil(L/4), d]; block b sums tokens 4b .. min(4b+3, L-1).

    [blog] "compresses keys into micro-blocks at compression ratio 4"; [pr]
    QSAIndexer.forward excerpt (raw keys pooled by the compress ratio into
    the compressed-key cache).  Pooling is read as a plain sum with no
    normalisation, so the indexer stays exact in integers.
    """
    k = np.asarray(k_idx, dtype=np.int64)
    L, d = k.shape
    n = num_blocks(L)
    # absent tokens of a partial tail block are zero rows: they add nothing
    padded = np.zeros((n * COMPRESS_RATIO, d), dtype=np.int64)
    padded[:L] = k
    return padded.reshape(n, COMPRESS_RATIO, d).sum(axis=1)


def block_scores(q_idx: np.ndarray, kc: np.ndarray, n_sel: int | None = None) -> np.ndarray:
    """Weight-free block score: integer dot product of the indexer query with
    each compressed key, for blocks 0 .. n_sel-1.

    [blog] "scores them"; [pr] "执行摘要" (weight-free top-k selection).
    """
    kc = np.asarray(kc, dtype=np.int64)
    if n_sel is None:
        n_sel = kc.shape[0]
    q = np.asarray(q_idx, dtype=np.int64)
    return kc[:n_sel] @ q


def select_blocks(scores: np.ndarray, topk: int = TOPK_BLOCKS) -> np.ndarray:
    """Keep the topk highest-scoring blocks.

    Order of preference: higher score first, then lower block index (the tie
    rule of the tiny workload).  The kept indices are returned ascending,
    padded with -1 to width topk ([pr] QSAIndexer.forward excerpt: fixed
    width, padded with -1).  int32 [topk].
    """
    s = np.asarray(scores, dtype=np.int64)
    n = s.shape[0]
    idx = np.arange(n, dtype=np.int64)
    order = np.lexsort((idx, -s))          # primary -s, secondary index
    keep = np.sort(order[: min(topk, n)])
    out = np.full(topk, -1, dtype=np.int32)
    out[: keep.shape[0]] = keep
    return out


def selection_width(L: int, T: int) -> int:
    """Blocks that compete for query token 0 at position p0 = L - T: those
    intersecting [0, p0], i.e. floor(p0/4) + 1.  For T = 1 this is
    ceil(L/4).  [pr] "实现拆解" (MTP step 0 selects, later steps reuse)."""
    p0 = int(L) - int(T)
    return p0 // COMPRESS_RATIO + 1


# ----------------------------------------------------------------------------
# Token sets and attention
# ----------------------------------------------------------------------------

def selection_tokens(sel: np.ndarray, L: int, T: int, budget: int) -> np.ndarray:
    """The selection as a token budget: the tokens of the selected blocks
    that query token 0 (position p0 = L - T) may see, i.e. positions <= p0,
    ascending, padded with -1 to width `budget`.  [pr] QSAIndexer.forward
    excerpt (the budget is a token count, token_topk = indexer_budget;
    forward returns fixed-width request-relative token indices padded with
    -1).  int32 [budget]."""
    p0 = int(L) - int(T)
    toks = sorted(4 * int(b) + j for b in np.asarray(sel) if b >= 0 for j in range(4)
                  if 4 * int(b) + j <= p0)
    out = np.full(int(budget), -1, dtype=np.int32)
    k = min(len(toks), int(budget))
    out[:k] = toks[:k]
    return out


def token_set(sel: np.ndarray, L: int, T: int, t: int) -> np.ndarray:
    """Token positions attended by query token t (position p_t = L - T + t).

    The union of the selected micro-blocks' tokens up to p_t and the
    speculative tail (p0, p_t], as a set (no token counted twice).  With
    T = 1 this is just the tokens of the selected blocks.  [blog] softmax
    over the selected tokens of the uncompressed K/V; [pr] MTP selection at
    step 0 reused by later steps.
    """
    p0 = L - T
    pt = p0 + t
    chosen = set()
    for b in np.asarray(sel).tolist():
        if b < 0:
            continue
        for i in range(COMPRESS_RATIO * b, COMPRESS_RATIO * b + COMPRESS_RATIO):
            if i <= pt:
                chosen.add(i)
    for i in range(p0 + 1, pt + 1):
        chosen.add(i)
    return np.array(sorted(chosen), dtype=np.int64)


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, tokens: np.ndarray,
              sm_scale: float) -> tuple[np.ndarray, np.ndarray]:
    """Exact softmax attention of one query token over a token subset.

    q: float64 [Hq, D]; K, V: float64 [L, Hkv, D]; tokens: int positions.
    Query head h reads kv head h // (Hq/Hkv) (grouped-query attention).
    Returns o float64 [Hq, D] and lse float64 [Hq] (natural log of the sum
    of exp of the scaled logits).  An empty token set gives o = 0 and
    lse = -inf.  [blog] "final softmax and value aggregation still run on
    the uncompressed K and V".
    """
    Hq, D = q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    o = np.zeros((Hq, D), dtype=np.float64)
    lse = np.full(Hq, -np.inf, dtype=np.float64)
    if tokens.shape[0] == 0:
        return o, lse
    for h in range(Hq):
        g = h // G
        x = sm_scale * (K[tokens, g, :] @ q[h])
        m = x.max()
        w = np.exp(x - m)
        z = w.sum()
        o[h] = (w / z) @ V[tokens, g, :]
        lse[h] = m + math.log(z)
    return o, lse


def split_bounds(L: int, page_size: int, num_splits: int) -> np.ndarray:
    """Split s owns logical pages [floor(s*NP/S), floor((s+1)*NP/S)),
    NP = ceil(L / page_size).  [blog] each decode-context-parallel rank
    reads only its own slice of the context.  Returned in token units:
    int64 [S+1] token boundaries (clipped to L)."""
    NP = (L + page_size - 1) // page_size
    pages = np.array([(s * NP) // num_splits for s in range(num_splits + 1)], dtype=np.int64)
    return np.minimum(pages * page_size, L)


def split_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, tokens: np.ndarray,
                    sm_scale: float, L: int, page_size: int, num_splits: int
                    ) -> tuple[np.ndarray, np.ndarray]:
    """Per-split partial attention: split s attends the tokens of its own
    page slice.  Returns o_part [S, Hq, D], lse_part [S, Hq]; an empty split
    gives o = 0, lse = -inf."""
    bounds = split_bounds(L, page_size, num_splits)
    Hq, D = q.shape
    o_part = np.zeros((num_splits, Hq, D), dtype=np.float64)
    lse_part = np.full((num_splits, Hq), -np.inf, dtype=np.float64)
    for s in range(num_splits):
        sub = tokens[(tokens >= bounds[s]) & (tokens < bounds[s + 1])]
        o_part[s], lse_part[s] = attention(q, K, V, sub, sm_scale)
    return o_part, lse_part


def lse_merge(o_part: np.ndarray, lse_part: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Log-sum-exp combine of partial attention results over axis 0.

    lse = log sum_s exp(lse_s);  o = sum_s exp(lse_s - lse) * o_s.
    All partials empty (-inf) -> o = 0, lse = -inf.  [blog] partial
    attention results are merged across ranks at the end.
    """
    o_part = np.asarray(o_part, dtype=np.float64)
    lse_part = np.asarray(lse_part, dtype=np.float64)
    m = lse_part.max(axis=0)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    w = np.where(np.isfinite(lse_part), np.exp(lse_part - m_safe[None]), 0.0)
    z = w.sum(axis=0)
    lse = np.where(finite, m_safe + np.log(np.where(finite, z, 1.0)), -np.inf)
    scale = np.where(finite[None], w / np.where(finite, z, 1.0)[None], 0.0)
    o = (scale[..., None] * o_part).sum(axis=0)
    return o, lse


# ----------------------------------------------------------------------------
# Paging helpers (plain indexing) and the whole per-request path
# ----------------------------------------------------------------------------

def depage(cache: np.ndarray, block_table_row: np.ndarray, L: int, page_size: int) -> np.ndarray:
    """Logical rows 0..L-1 of a paged cache [num_pages, page_size, ...]."""
    npg = (L + page_size - 1) // page_size
    pages = np.asarray(block_table_row[:npg], dtype=np.int64)
    flat = cache[pages].reshape((npg * page_size,) + cache.shape[2:])
    return flat[:L]


def depage_kc(kc_cache: np.ndarray, block_table_row: np.ndarray, L: int, page_size: int) -> np.ndarray:
    """Logical compressed keys of blocks 0..ceil(L/4)-1 from the paged
    compressed-key cache [num_pages, page_size/4, d] (indexed by the same
    block table as K/V)."""
    bpp = page_size // COMPRESS_RATIO
    n = num_blocks(L)
    npg = (n + bpp - 1) // bpp
    pages = np.asarray(block_table_row[:npg], dtype=np.int64)
    flat = kc_cache[pages].reshape((npg * bpp,) + kc_cache.shape[2:])
    return flat[:n]


def decode_request(k_idx: np.ndarray, q_idx: np.ndarray, q: np.ndarray, K: np.ndarray,
                   V: np.ndarray, T: int, page_size: int, num_splits: int,
                   topk: int = TOPK_BLOCKS, sm_scale: float | None = None) -> dict:
    """The whole decode path for one request, from logical inputs.

    k_idx int8 [L, d]; q_idx int8 [d] (indexer query of token 0);
    q float64 [T, Hq, D]; K, V float64 [L, Hkv, D] (already dequantised).
    K and V may also be StoredRows views (decoded row by row on access).
    Returns kc, scores, sel, per-token o/lse (unsplit), o_part/lse_part per
    split and the merged o/lse.
    """
    L = k_idx.shape[0]
    D = q.shape[-1]
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    kc = compress_keys(k_idx)
    n_sel = selection_width(L, T)
    scores = block_scores(q_idx, kc, n_sel)
    sel = select_blocks(scores, topk)
    Hq = q.shape[1]
    o = np.zeros((T, Hq, D))
    lse = np.zeros((T, Hq))
    o_part = np.zeros((num_splits, T, Hq, D))
    lse_part = np.zeros((num_splits, T, Hq))
    for t in range(T):
        toks = token_set(sel, L, T, t)
        o[t], lse[t] = attention(q[t], K, V, toks, sm_scale)
        o_part[:, t], lse_part[:, t] = split_attention(q[t], K, V, toks, sm_scale, L,
                                                       page_size, num_splits)
    o_m, lse_m = lse_merge(o_part, lse_part)
    return dict(kc=kc, scores=scores, sel=sel, o=o, lse=lse, o_part=o_part,
                lse_part=lse_part, o_merged=o_m, lse_merged=lse_m)
