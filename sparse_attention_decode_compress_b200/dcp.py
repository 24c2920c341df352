"""Decode context parallelism (DCP) over torch.distributed.

Each rank holds one slice of every request's KV pages.  The selector
(compressed-key cache, raw-key ring, selection) is replicated, so every rank
runs the same qsa_compress_append and qsa_index_topk.  Rank k then attends
only the selected tokens of its own slice: split k of S = world size, with
split s owning logical pages [floor(s*NP/S), floor((s+1)*NP/S)).  The
per-rank partial results (o_s, lse_s) are all-gathered and merged by
log-sum-exp with qsa_lse_merge.  (Blog "Qwen 4 QSA 迎来解码上下文并行…",
section 拉取请求实际改变了什么: each DCP rank reads its own slice of the
cache and the partial results are merged; the selector and side caches are
replicated.)

The exchange is one all-gather of B*T*Hq*(D+1) floats per rank and step
(1 MiB at batch 128, 16 query heads, head dim 128).
"""
from __future__ import annotations

import math

import torch
import torch.distributed as dist

from .api import (QSACache, new_workspace, qsa_lse_merge, qsa_sparse_decode_splits,
                  qsa_sparse_decode_workspace_bytes)


def dcp_exchange(o_local: torch.Tensor, lse_local: torch.Tensor, o_all: torch.Tensor,
                 lse_all: torch.Tensor, group=None) -> None:
    """All-gathers every rank's split partials: after the call o_all[k] and
    lse_all[k] hold rank k's o_local[0] and lse_local[0] (shapes
    [1, ...] -> [world, ...])."""
    world = dist.get_world_size(group)
    if o_all.shape[0] != world or lse_all.shape[0] != world:
        raise ValueError("o_all and lse_all need one slot per rank")
    dist.all_gather(list(o_all.unbind(0)), o_local[0], group=group)
    dist.all_gather(list(lse_all.unbind(0)), lse_local[0], group=group)


class DCPDecode:
    """One DCP decode step after the replicated selection: this rank's split
    (qsa_sparse_decode_splits), the exchange, and the merge."""

    def __init__(self, cache: QSACache, B: int, T: int, Hq: int, topk: int, group=None,
                 device=None):
        device = device or cache.k_cache.device
        _, _, Hkv, D = cache.k_cache.shape
        self.cache, self.group = cache, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.sm_scale = 1.0 / math.sqrt(D)
        self.o_local = torch.empty((1, B, T, Hq, D), dtype=torch.float32, device=device)
        self.lse_local = torch.empty((1, B, T, Hq), dtype=torch.float32, device=device)
        self.o_all = torch.empty((self.world, B, T, Hq, D), dtype=torch.float32, device=device)
        self.lse_all = torch.empty((self.world, B, T, Hq), dtype=torch.float32, device=device)
        self.o = torch.empty((B, T, Hq, D), dtype=torch.float32, device=device)
        self.lse = torch.empty((B, T, Hq), dtype=torch.float32, device=device)
        self.ws = new_workspace(
            qsa_sparse_decode_workspace_bytes(B, T, Hq, Hkv, D, topk, self.world), device)

    def __call__(self, q: torch.Tensor, ctx_lens: torch.Tensor, sel: torch.Tensor, stream=None):
        qsa_sparse_decode_splits(self.cache, q, ctx_lens, sel, self.sm_scale, self.world, self.rank,
                                 self.rank + 1, self.o_local, self.lse_local, self.ws, stream)
        dcp_exchange(self.o_local, self.lse_local, self.o_all, self.lse_all, self.group)
        qsa_lse_merge(self.o_all, self.lse_all, self.o, self.lse, stream)
        return self.o, self.lse
