"""Decode-time Qwen Sparse Attention (QSA) on B200: a C-ABI library of
hand-written sm_100a kernels (libqsa.so) and its thin PyTorch binding."""
from .api import (QSACache, QSAError, QSASession, allocate_norm_caches, new_workspace,
                  qsa_compress_append, qsa_compress_append_norm, qsa_index_topk_norm,
                  qsa_kcn_page_bytes, qsa_sparse_prefill, qsa_sparse_prefill_workspace_bytes,
                  qsa_get_device_error, qsa_index_topk, qsa_index_topk_noalloc,
                  qsa_index_topk_tokens, qsa_index_topk_workspace_bytes, qsa_lse_merge,
                  qsa_sparse_decode, qsa_sparse_decode_merged, qsa_sparse_decode_splits,
                  qsa_sparse_decode_workspace_bytes)
from .dcp import DCPDecode, dcp_exchange
from .decode import QSADecodeStep, QSADraftDecode

__all__ = [
    "DCPDecode", "QSACache", "QSAError", "QSADecodeStep", "QSADraftDecode", "QSASession", "dcp_exchange",
    "allocate_norm_caches", "new_workspace", "qsa_compress_append", "qsa_compress_append_norm",
    "qsa_index_topk_norm", "qsa_kcn_page_bytes", "qsa_sparse_prefill",
    "qsa_sparse_prefill_workspace_bytes",
    "qsa_get_device_error", "qsa_index_topk", "qsa_index_topk_noalloc", "qsa_index_topk_tokens",
    "qsa_index_topk_workspace_bytes", "qsa_lse_merge",
    "qsa_sparse_decode", "qsa_sparse_decode_merged", "qsa_sparse_decode_splits",
    "qsa_sparse_decode_workspace_bytes",
]
