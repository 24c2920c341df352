"""One decode step of the QSA hot path through the C ABI:
compress-append -> index top-k -> sparse split-KV decode and the LSE merge
of its splits (qsa_sparse_decode_merged: two kernels).  Holds the step's output buffers
and workspaces; every step is a kernel."""
from __future__ import annotations

import math

import torch

from .api import (QSACache, new_workspace, qsa_compress_append, qsa_index_topk,
                  qsa_index_topk_tokens, qsa_index_topk_workspace_bytes,
                  qsa_sparse_decode_merged, qsa_sparse_decode_workspace_bytes)


class QSADecodeStep:
    def __init__(self, cache: QSACache, B: int, T: int, Hq: int, topk: int, num_splits: int,
                 max_blocks: int, device=None, keep_scores: bool = False):
        device = device or cache.k_cache.device
        _, _, Hkv, D = cache.k_cache.shape
        self.cache, self.B, self.T, self.Hq, self.D = cache, B, T, Hq, D
        self.topk, self.S, self.max_blocks = topk, num_splits, max_blocks
        self.sm_scale = 1.0 / math.sqrt(D)
        self.sel = torch.empty((B, topk), dtype=torch.int32, device=device)
        self.scores = (torch.empty((B, max_blocks), dtype=torch.int32, device=device)
                       if keep_scores else None)
        self.o_part = torch.empty((num_splits, B, T, Hq, D), dtype=torch.float32, device=device)
        self.lse_part = torch.empty((num_splits, B, T, Hq), dtype=torch.float32, device=device)
        self.o = torch.empty((B, T, Hq, D), dtype=torch.float32, device=device)
        self.lse = torch.empty((B, T, Hq), dtype=torch.float32, device=device)
        self.ws_topk = new_workspace(qsa_index_topk_workspace_bytes(B, max_blocks), device)
        self.ws_dec = new_workspace(
            qsa_sparse_decode_workspace_bytes(B, T, Hq, Hkv, D, topk, num_splits), device)

    def __call__(self, pos0, cu_new, k_new, q_idx, q, ctx_lens, n_sel=None, stream=None):
        qsa_compress_append(self.cache, pos0, cu_new, k_new, self.T, stream)
        qsa_index_topk(self.cache, q_idx, ctx_lens, n_sel, self.max_blocks, self.topk, self.sel,
                       self.scores, self.ws_topk, stream)
        qsa_sparse_decode_merged(self.cache, q, ctx_lens, self.sel, self.sm_scale, self.S,
                                 self.o_part, self.lse_part, self.o, self.lse, self.ws_dec, stream)
        return self.o, self.lse

    @property
    def kernels_per_step(self) -> int:
        """Kernels one step launches: append, scan, select, then the decode
        and its merge; the chunked decode (float32 or fp8 caches) adds the
        kernel that zeroes its workspace header."""
        chunked = self.cache.k_cache.dtype != torch.bfloat16
        return 6 if chunked else 5


class QSADraftDecode:
    """Multi-step MTP drafting with one indexer run: the selecting step picks
    the blocks for its query token, and the draft steps after it reuse that
    selection while still appending their keys to the side caches (PR
    #53896 report, QSAIndexer.forward excerpt: with skip_topk the indexer
    returns the buffer filled by MTP step 0 and only updates the raw-key
    ring and compressed-key caches).

    select(): the selecting step, at position p0 = ctx_lens - 1 of each
      request: qsa_compress_append of its indexer key,
      qsa_index_topk_tokens (the token rows, the buffer later steps reuse,
      and the kept blocks), then the decode of query row 0 (T = 1).
    draft(): draft step k = 1, 2, ... (at most max_draft): appends the draft
      token's indexer key at p0 + k, then decodes with the kept blocks.
      Draft token k attends the kept blocks' tokens up to p0 + k and every
      token after p0, which is query row k of an MTP decode with T = k + 1
      on the same selection, so it is that call (rows 0 .. k-1 are
      recomputed and dropped).  ctx_lens = p0 + k + 1 and q holds the
      queries of steps 0 .. k.
    Both return (token rows [B, budget], o [B, Hq, D], lse [B, Hq]) views
    of the driver's buffers.  Every step is a library call."""

    def __init__(self, cache: QSACache, B: int, Hq: int, budget: int, num_splits: int,
                 max_blocks: int, max_draft: int = 3, device=None):
        device = device or cache.k_cache.device
        _, _, Hkv, D = cache.k_cache.shape
        if budget % 4 != 0 or not 1 <= max_draft <= 3:
            raise ValueError("budget must be a multiple of 4 and max_draft in 1..3")
        self.cache, self.B, self.Hq, self.D = cache, B, Hq, D
        self.budget, self.topk, self.S = budget, budget // 4, num_splits
        self.max_blocks, self.max_draft = max_blocks, max_draft
        self.sm_scale = 1.0 / math.sqrt(D)
        self.tokens = torch.empty((B, budget), dtype=torch.int32, device=device)
        self.sel = torch.empty((B, self.topk), dtype=torch.int32, device=device)
        self.cu1 = torch.arange(0, B + 1, dtype=torch.int32, device=device)
        T = max_draft + 1
        self.o_part = [torch.empty((num_splits, B, t, Hq, D), dtype=torch.float32, device=device)
                       for t in range(1, T + 1)]
        self.lse_part = [torch.empty((num_splits, B, t, Hq), dtype=torch.float32, device=device)
                         for t in range(1, T + 1)]
        self.o = [torch.empty((B, t, Hq, D), dtype=torch.float32, device=device)
                  for t in range(1, T + 1)]
        self.lse = [torch.empty((B, t, Hq), dtype=torch.float32, device=device)
                    for t in range(1, T + 1)]
        self.ws_topk = new_workspace(qsa_index_topk_workspace_bytes(B, max_blocks), device)
        self.ws_dec = new_workspace(
            qsa_sparse_decode_workspace_bytes(B, T, Hq, Hkv, D, self.topk, num_splits), device)
        self.k = -1

    def select(self, pos0, k_new, q_idx, q, ctx_lens, stream=None):
        qsa_compress_append(self.cache, pos0, self.cu1, k_new, 1, stream)
        qsa_index_topk_tokens(self.cache, q_idx, ctx_lens, None, 1, self.max_blocks, self.budget,
                              self.tokens, self.sel, None, self.ws_topk, stream)
        qsa_sparse_decode_merged(self.cache, q, ctx_lens, self.sel, self.sm_scale, self.S,
                                 self.o_part[0], self.lse_part[0], self.o[0], self.lse[0],
                                 self.ws_dec, stream)
        self.k = 0
        return self.tokens, self.o[0][:, 0], self.lse[0][:, 0]

    def draft(self, pos, k_new, q, ctx_lens, stream=None):
        if self.k < 0:
            raise RuntimeError("draft() needs a select() first: there is no selection to reuse")
        k = self.k + 1
        if k > self.max_draft:
            raise RuntimeError(f"at most {self.max_draft} draft steps reuse one selection")
        if q.shape[1] != k + 1:
            raise ValueError(f"draft step {k} takes the queries of steps 0..{k}: q[:, {k + 1}]")
        qsa_compress_append(self.cache, pos, self.cu1, k_new, 1, stream)
        qsa_sparse_decode_merged(self.cache, q, ctx_lens, self.sel, self.sm_scale, self.S,
                                 self.o_part[k], self.lse_part[k], self.o[k], self.lse[k],
                                 self.ws_dec, stream)
        self.k = k
        return self.tokens, self.o[k][:, k], self.lse[k][:, k]
