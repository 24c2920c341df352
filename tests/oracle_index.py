"""The oracle's indexer path for one request (compress -> score -> select),
in a module that imports nothing but NumPy and the oracle, so that a pool
of `spawn` worker processes can run it next to the GPU tests.  Test
infrastructure only."""
from __future__ import annotations

import os
from concurrent.futures import ProcessPoolExecutor
import multiprocessing as mp

import numpy as np

from oracle import qsa_ref as ref


def index_request(k_idx: np.ndarray, q_idx: np.ndarray, T: int, topk: int):
    """Scores of the competing blocks and the selection row of one request
    whose raw indexer keys (logical order) are k_idx [L, d]."""
    L = k_idx.shape[0]
    kc = ref.compress_keys(k_idx)
    scores = ref.block_scores(q_idx, kc, ref.selection_width(L, T))
    return scores, ref.select_blocks(scores, topk)


def pool_size(max_workers: int = 16) -> int:
    return max(1, min(max_workers, len(os.sched_getaffinity(0))))


def pool(workers: int) -> ProcessPoolExecutor:
    """A process pool started with `spawn` (safe to start after CUDA is
    initialised in the parent)."""
    return ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn"))
