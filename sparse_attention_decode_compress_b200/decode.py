"""One decode step of the QSA hot path through the C ABI:
compress-append -> index top-k -> sparse split-KV decode and the LSE merge
of its splits (qsa_sparse_decode_merged: two kernels).  Holds the step's output buffers
and workspaces; every step is a kernel."""
from __future__ import annotations

import math

import torch

from .api import (QSACache, new_workspace, qsa_compress_append, qsa_index_topk,
                  qsa_index_topk_workspace_bytes, qsa_sparse_decode_merged,
                  qsa_sparse_decode_workspace_bytes)


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

    # kernels one call launches: append, scan, select, decode, merge
    kernels_per_step = 5
