"""Thin PyTorch binding of libqsa.so.

The functions carry the names of the C entry points and do argument
marshalling only: they check dtypes, shapes and contiguity on the host, pass
raw device pointers and the current CUDA stream, and raise on a non-OK
status.  Every step of the computation runs in the CUDA kernels; PyTorch only
owns device memory and streams.  There is no CPU path.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib

_KV_DTYPES = {torch.float32: _lib.QSA_F32, torch.bfloat16: _lib.QSA_BF16,
              torch.float8_e4m3fn: _lib.QSA_FP8_E4M3}


class QSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = _lib.load()
        super().__init__(f"{where}: {lib.qsa_status_string(status).decode()}")
        self.status = status


def _check(status: int, where: str):
    if status != _lib.QSA_OK:
        raise QSAError(status, where)


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to libqsa must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("tensors passed to libqsa must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int | None:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _need(t: torch.Tensor, dtype, name: str):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


@dataclass
class QSACache:
    """One attention layer's paged caches (a single cache group: the same
    block-table entry names the same physical page in K, V and the
    compressed-key cache)."""
    k_cache: torch.Tensor               # [num_pages, P, Hkv, D] f32 / bf16 / fp8 e4m3
    v_cache: torch.Tensor
    kc: torch.Tensor                    # uint8 [num_pages, qsa_kc_page_bytes(P, d)], packed
    ring: torch.Tensor                  # int8 [ring_rows, 4, d]
    block_table: torch.Tensor           # int32 [B, max_pages]
    k_scale: torch.Tensor | None = None  # f32 [num_pages, Hkv] (fp8 only)
    v_scale: torch.Tensor | None = None

    @staticmethod
    def allocate(k_cache, v_cache, block_table, idx_dim: int, ring_rows: int,
                 k_scale=None, v_scale=None) -> "QSACache":
        num_pages, P = k_cache.shape[0], k_cache.shape[1]
        page_bytes = int(_lib.load().qsa_kc_page_bytes(P, idx_dim))
        if page_bytes == 0:
            raise ValueError(f"unsupported compressed-key geometry: page_size {P}, idx_dim {idx_dim}")
        kc = torch.zeros((num_pages, page_bytes), dtype=torch.uint8, device=k_cache.device)
        ring = torch.zeros((ring_rows, 4, idx_dim), dtype=torch.int8, device=k_cache.device)
        return QSACache(k_cache, v_cache, kc, ring, block_table, k_scale, v_scale)

    def struct(self) -> _lib.QsaCacheStruct:
        k, v = self.k_cache, self.v_cache
        if k.dtype not in _KV_DTYPES or v.dtype != k.dtype or k.shape != v.shape or k.dim() != 4:
            raise TypeError("k_cache / v_cache must be [num_pages, P, Hkv, D] of one dtype "
                            "(float32, bfloat16 or float8_e4m3fn)")
        _need(self.kc, torch.uint8, "kc")
        _need(self.ring, torch.int8, "ring")
        _need(self.block_table, torch.int32, "block_table")
        num_pages, P, Hkv, D = k.shape
        d = self.ring.shape[-1]
        page_bytes = int(_lib.load().qsa_kc_page_bytes(P, d))
        if self.ring.dim() != 3 or self.ring.shape[1] != 4 or page_bytes == 0 or \
                self.kc.shape != (num_pages, page_bytes):
            raise ValueError("ring must be [rows, 4, d] and kc [num_pages, qsa_kc_page_bytes(P, d)]")
        s = _lib.QsaCacheStruct()
        s.num_pages, s.page_size, s.num_kv_heads, s.head_dim, s.idx_dim = num_pages, P, Hkv, D, d
        s.kv_dtype = _KV_DTYPES[k.dtype]
        s.k_cache, s.v_cache = _ptr(k), _ptr(v)
        s.k_scale, s.v_scale = _ptr(self.k_scale), _ptr(self.v_scale)
        s.kc, s.ring = _ptr(self.kc), _ptr(self.ring)
        s.ring_rows = self.ring.shape[0]
        s.block_table = _ptr(self.block_table)
        s.max_pages_per_req = self.block_table.shape[1]
        return s


def qsa_compress_append(cache: QSACache, pos0: torch.Tensor, cu_new: torch.Tensor,
                        k_new: torch.Tensor, max_new_per_req: int, stream=None) -> None:
    _need(pos0, torch.int32, "pos0")
    _need(cu_new, torch.int32, "cu_new")
    _need(k_new, torch.int8, "k_new")
    B = pos0.shape[0]
    if cu_new.shape[0] != B + 1:
        raise ValueError("cu_new must have B+1 entries")
    s = cache.struct()
    lib = _lib.load()
    _check(lib.qsa_compress_append(ctypes.byref(s), B, _ptr(pos0), _ptr(cu_new), _ptr(k_new),
                                   int(max_new_per_req), _stream(stream)), "qsa_compress_append")


def qsa_index_topk_workspace_bytes(B: int, max_blocks: int) -> int:
    return int(_lib.load().qsa_index_topk_workspace_bytes(B, max_blocks))


def qsa_sparse_decode_workspace_bytes(B: int, T: int, Hq: int, Hkv: int, D: int, topk: int,
                                      num_splits: int) -> int:
    return int(_lib.load().qsa_sparse_decode_workspace_bytes(B, T, Hq, Hkv, D, topk, num_splits))


def new_workspace(nbytes: int, device) -> torch.Tensor:
    """Workspace buffer (zero-filled; no call needs it zeroed: the stream-K
    decode keeps no state between calls and the chunked decode zeroes its
    header in every call)."""
    return torch.zeros(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def qsa_index_topk(cache: QSACache, q_idx: torch.Tensor, ctx_lens: torch.Tensor,
                   n_sel: torch.Tensor | None, max_blocks: int, topk: int, sel: torch.Tensor,
                   scores: torch.Tensor | None, workspace: torch.Tensor, stream=None) -> None:
    _need(q_idx, torch.int8, "q_idx")
    _need(ctx_lens, torch.int32, "ctx_lens")
    _need(sel, torch.int32, "sel")
    B = q_idx.shape[0]
    if sel.shape != (B, topk):
        raise ValueError("sel must be [B, topk]")
    if n_sel is not None:
        _need(n_sel, torch.int32, "n_sel")
    if scores is not None:
        _need(scores, torch.int32, "scores")
        if scores.shape != (B, max_blocks):
            raise ValueError("scores must be [B, max_blocks]")
    s = cache.struct()
    lib = _lib.load()
    _check(lib.qsa_index_topk(ctypes.byref(s), B, _ptr(q_idx), _ptr(ctx_lens), _ptr(n_sel),
                              int(max_blocks), int(topk), _ptr(sel), _ptr(scores),
                              _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream(stream)), "qsa_index_topk")


def qsa_index_topk_noalloc(cache: QSACache, q_idx: torch.Tensor, ctx_lens: torch.Tensor,
                           n_sel: torch.Tensor | None, max_blocks: int, topk: int,
                           sel: torch.Tensor, stream=None) -> None:
    """qsa_index_topk for callers that cannot provide a workspace: the
    scores live in a fixed 32 MiB array inside libqsa.so (B * max_blocks
    must not exceed 8,388,608)."""
    _need(q_idx, torch.int8, "q_idx")
    _need(ctx_lens, torch.int32, "ctx_lens")
    _need(sel, torch.int32, "sel")
    B = q_idx.shape[0]
    if sel.shape != (B, topk):
        raise ValueError("sel must be [B, topk]")
    if n_sel is not None:
        _need(n_sel, torch.int32, "n_sel")
    s = cache.struct()
    lib = _lib.load()
    _check(lib.qsa_index_topk_noalloc(ctypes.byref(s), B, _ptr(q_idx), _ptr(ctx_lens), _ptr(n_sel),
                                      int(max_blocks), int(topk), _ptr(sel), _stream(stream)),
           "qsa_index_topk_noalloc")


def qsa_index_topk_tokens(cache: QSACache, q_idx: torch.Tensor, ctx_lens: torch.Tensor,
                          n_sel: torch.Tensor | None, T: int, max_blocks: int, budget: int,
                          tokens: torch.Tensor, sel: torch.Tensor | None,
                          scores: torch.Tensor | None, workspace: torch.Tensor,
                          stream=None) -> None:
    """The selection as fixed-width rows of token indices ([B, budget],
    -1 padded); `sel` ([B, budget // 4]) optionally receives the blocks."""
    _need(q_idx, torch.int8, "q_idx")
    _need(ctx_lens, torch.int32, "ctx_lens")
    _need(tokens, torch.int32, "tokens")
    B = q_idx.shape[0]
    if tokens.shape != (B, budget):
        raise ValueError("tokens must be [B, budget]")
    if sel is not None:
        _need(sel, torch.int32, "sel")
        if sel.shape != (B, budget // 4):
            raise ValueError("sel must be [B, budget // 4]")
    if n_sel is not None:
        _need(n_sel, torch.int32, "n_sel")
    if scores is not None:
        _need(scores, torch.int32, "scores")
        if scores.shape != (B, max_blocks):
            raise ValueError("scores must be [B, max_blocks]")
    s = cache.struct()
    lib = _lib.load()
    _check(lib.qsa_index_topk_tokens(ctypes.byref(s), B, _ptr(q_idx), _ptr(ctx_lens), _ptr(n_sel),
                                     int(T), int(max_blocks), int(budget), _ptr(tokens), _ptr(sel),
                                     _ptr(scores), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(stream)),
           "qsa_index_topk_tokens")


def qsa_sparse_decode(cache: QSACache, q: torch.Tensor, ctx_lens: torch.Tensor,
                      sel: torch.Tensor, sm_scale: float, num_splits: int,
                      o_part: torch.Tensor, lse_part: torch.Tensor, workspace: torch.Tensor,
                      stream=None) -> None:
    B, T, Hq, D = q.shape
    q_dt = {torch.float32: _lib.QSA_F32, torch.bfloat16: _lib.QSA_BF16}.get(q.dtype)
    if q_dt is None:
        raise TypeError("q must be float32 or bfloat16")
    _need(ctx_lens, torch.int32, "ctx_lens")
    _need(sel, torch.int32, "sel")
    _need(o_part, torch.float32, "o_part")
    _need(lse_part, torch.float32, "lse_part")
    if o_part.shape != (num_splits, B, T, Hq, D) or lse_part.shape != (num_splits, B, T, Hq):
        raise ValueError("o_part must be [S, B, T, Hq, D] and lse_part [S, B, T, Hq]")
    s = cache.struct()
    lib = _lib.load()
    _check(lib.qsa_sparse_decode(ctypes.byref(s), B, T, Hq, _ptr(q), q_dt, _ptr(ctx_lens),
                                 _ptr(sel), sel.shape[1], float(sm_scale), int(num_splits),
                                 _ptr(o_part), _ptr(lse_part), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)),
           "qsa_sparse_decode")


def qsa_sparse_decode_merged(cache: QSACache, q: torch.Tensor, ctx_lens: torch.Tensor,
                             sel: torch.Tensor, sm_scale: float, num_splits: int,
                             o_part: torch.Tensor, lse_part: torch.Tensor, o: torch.Tensor,
                             lse: torch.Tensor, workspace: torch.Tensor, stream=None) -> None:
    """qsa_sparse_decode and the split merge in one call (o / lse as
    qsa_lse_merge of o_part / lse_part; two kernels)."""
    B, T, Hq, D = q.shape
    q_dt = {torch.float32: _lib.QSA_F32, torch.bfloat16: _lib.QSA_BF16}.get(q.dtype)
    if q_dt is None:
        raise TypeError("q must be float32 or bfloat16")
    for t, n in ((o_part, "o_part"), (lse_part, "lse_part"), (o, "o"), (lse, "lse")):
        _need(t, torch.float32, n)
    _need(ctx_lens, torch.int32, "ctx_lens")
    _need(sel, torch.int32, "sel")
    if o_part.shape != (num_splits, B, T, Hq, D) or lse_part.shape != (num_splits, B, T, Hq):
        raise ValueError("o_part must be [S, B, T, Hq, D] and lse_part [S, B, T, Hq]")
    if o.shape != (B, T, Hq, D) or lse.shape != (B, T, Hq):
        raise ValueError("o must be [B, T, Hq, D] and lse [B, T, Hq]")
    s = cache.struct()
    lib = _lib.load()
    _check(lib.qsa_sparse_decode_merged(ctypes.byref(s), B, T, Hq, _ptr(q), q_dt, _ptr(ctx_lens),
                                        _ptr(sel), sel.shape[1], float(sm_scale), int(num_splits),
                                        _ptr(o_part), _ptr(lse_part), _ptr(o), _ptr(lse),
                                        _ptr(workspace),
                                        workspace.numel() * workspace.element_size(),
                                        _stream(stream)),
           "qsa_sparse_decode_merged")


def qsa_sparse_decode_splits(cache: QSACache, q: torch.Tensor, ctx_lens: torch.Tensor,
                             sel: torch.Tensor, sm_scale: float, num_splits: int, split_lo: int,
                             split_hi: int, o_part: torch.Tensor, lse_part: torch.Tensor,
                             workspace: torch.Tensor, stream=None) -> None:
    """Splits [split_lo, split_hi) of num_splits only; o_part / lse_part
    hold them from index 0 ([split_hi - split_lo, ...])."""
    B, T, Hq, D = q.shape
    q_dt = {torch.float32: _lib.QSA_F32, torch.bfloat16: _lib.QSA_BF16}.get(q.dtype)
    if q_dt is None:
        raise TypeError("q must be float32 or bfloat16")
    _need(ctx_lens, torch.int32, "ctx_lens")
    _need(sel, torch.int32, "sel")
    _need(o_part, torch.float32, "o_part")
    _need(lse_part, torch.float32, "lse_part")
    n = split_hi - split_lo
    if o_part.shape != (n, B, T, Hq, D) or lse_part.shape != (n, B, T, Hq):
        raise ValueError("o_part must be [split_hi - split_lo, B, T, Hq, D] and lse_part "
                         "[split_hi - split_lo, B, T, Hq]")
    s = cache.struct()
    lib = _lib.load()
    _check(lib.qsa_sparse_decode_splits(ctypes.byref(s), B, T, Hq, _ptr(q), q_dt, _ptr(ctx_lens),
                                        _ptr(sel), sel.shape[1], float(sm_scale), int(num_splits),
                                        int(split_lo), int(split_hi), _ptr(o_part), _ptr(lse_part),
                                        _ptr(workspace),
                                        workspace.numel() * workspace.element_size(),
                                        _stream(stream)),
           "qsa_sparse_decode_splits")


def qsa_lse_merge(o_part: torch.Tensor, lse_part: torch.Tensor, o: torch.Tensor,
                  lse: torch.Tensor, stream=None) -> None:
    for t, n in ((o_part, "o_part"), (lse_part, "lse_part"), (o, "o"), (lse, "lse")):
        _need(t, torch.float32, n)
    S, D = o_part.shape[0], o_part.shape[-1]
    rows = lse_part[0].numel()
    if o_part.numel() != S * rows * D or o.numel() != rows * D or lse.numel() != rows:
        raise ValueError("shapes of o_part [S, rows, D], lse_part [S, rows], o [rows, D], lse [rows]")
    lib = _lib.load()
    _check(lib.qsa_lse_merge(S, rows, D, _ptr(o_part), _ptr(lse_part), _ptr(o), _ptr(lse),
                             _stream(stream)), "qsa_lse_merge")


def qsa_kcn_page_bytes(page_size: int, idx_dim: int) -> int:
    return int(_lib.load().qsa_kcn_page_bytes(page_size, idx_dim))


def allocate_norm_caches(cache: QSACache, ring_rows: int) -> tuple[torch.Tensor, torch.Tensor]:
    """Side caches of the normalised-pooling indexer, in the cache group of
    `cache` (its block table names their pages): float16 compressed keys
    [num_pages, P/4, d] and the bfloat16 raw-key ring [ring_rows, 4, d]."""
    num_pages, P = cache.k_cache.shape[0], cache.k_cache.shape[1]
    d = cache.ring.shape[-1]
    if qsa_kcn_page_bytes(P, d) == 0:
        raise ValueError(f"unsupported compressed-key geometry: page_size {P}, idx_dim {d}")
    dev = cache.k_cache.device
    kcn = torch.zeros((num_pages, P // 4, d), dtype=torch.float16, device=dev)
    ring = torch.zeros((ring_rows, 4, d), dtype=torch.bfloat16, device=dev)
    return kcn, ring


def _check_norm_caches(cache: QSACache, kcn: torch.Tensor, ring: torch.Tensor):
    num_pages, P = cache.k_cache.shape[0], cache.k_cache.shape[1]
    d = cache.ring.shape[-1]
    _need(kcn, torch.float16, "kcn")
    _need(ring, torch.bfloat16, "ring")
    if tuple(kcn.shape) != (num_pages, P // 4, d) or ring.dim() != 3 or ring.shape[1:] != (4, d):
        raise ValueError("kcn must be [num_pages, P/4, d] float16 and ring [rows, 4, d] bfloat16")


def qsa_compress_append_norm(cache: QSACache, kcn: torch.Tensor, ring: torch.Tensor,
                             norm_weight: torch.Tensor | None, eps: float, pos0: torch.Tensor,
                             cu_new: torch.Tensor, k_new: torch.Tensor, max_new_per_req: int,
                             stream=None) -> None:
    """Normalised-pooling compress-append: bfloat16 raw keys k_new [N, d]
    into the ring and the float16 compressed-key pages."""
    _check_norm_caches(cache, kcn, ring)
    _need(pos0, torch.int32, "pos0")
    _need(cu_new, torch.int32, "cu_new")
    _need(k_new, torch.bfloat16, "k_new")
    if norm_weight is not None:
        _need(norm_weight, torch.float32, "norm_weight")
    B = pos0.shape[0]
    if cu_new.shape[0] != B + 1:
        raise ValueError("cu_new must have B+1 entries")
    s = cache.struct()
    s.ring_rows = ring.shape[0]
    _check(_lib.load().qsa_compress_append_norm(ctypes.byref(s), _ptr(kcn), _ptr(ring),
                                                _ptr(norm_weight), float(eps), B, _ptr(pos0),
                                                _ptr(cu_new), _ptr(k_new), int(max_new_per_req),
                                                _stream(stream)), "qsa_compress_append_norm")


def qsa_index_topk_norm(cache: QSACache, kcn: torch.Tensor, q_idx: torch.Tensor,
                        ctx_lens: torch.Tensor, n_sel: torch.Tensor | None, max_blocks: int,
                        topk: int, sel: torch.Tensor, scores: torch.Tensor | None,
                        workspace: torch.Tensor, stream=None) -> None:
    """Float scores of the normalised compressed keys against the bfloat16
    indexer query q_idx [B, d], and the top-k selection on them."""
    _need(kcn, torch.float16, "kcn")
    _need(q_idx, torch.bfloat16, "q_idx")
    _need(ctx_lens, torch.int32, "ctx_lens")
    _need(sel, torch.int32, "sel")
    B = q_idx.shape[0]
    if sel.shape != (B, topk):
        raise ValueError("sel must be [B, topk]")
    if n_sel is not None:
        _need(n_sel, torch.int32, "n_sel")
    if scores is not None:
        _need(scores, torch.float32, "scores")
        if scores.shape != (B, max_blocks):
            raise ValueError("scores must be [B, max_blocks]")
    s = cache.struct()
    _check(_lib.load().qsa_index_topk_norm(ctypes.byref(s), _ptr(kcn), B, _ptr(q_idx),
                                           _ptr(ctx_lens), _ptr(n_sel), int(max_blocks), int(topk),
                                           _ptr(sel), _ptr(scores), _ptr(workspace),
                                           workspace.numel() * workspace.element_size(),
                                           _stream(stream)), "qsa_index_topk_norm")


def qsa_sparse_prefill_workspace_bytes(n_tokens: int, max_blocks: int, Hq: int, Hkv: int, D: int,
                                       topk: int) -> int:
    return int(_lib.load().qsa_sparse_prefill_workspace_bytes(n_tokens, max_blocks, Hq, Hkv, D,
                                                              topk))


def qsa_sparse_prefill(cache: QSACache, cu_q: torch.Tensor, ctx_lens: torch.Tensor,
                       max_q_per_req: int, q_idx: torch.Tensor, k_chunk: torch.Tensor,
                       q: torch.Tensor, max_blocks: int, topk: int, sm_scale: float,
                       sel: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
                       workspace: torch.Tensor, stream=None) -> None:
    """Sparse prefill of the newest n_r tokens of each request (rows cu_q[r]
    .. cu_q[r+1]-1): every token selects its own blocks over its prefix and
    attends them.  q [Nq, Hq, D], q_idx / k_chunk [Nq, d] int8, sel
    [Nq, topk], o [Nq, Hq, D], lse [Nq, Hq]."""
    Nq, Hq, D = q.shape
    q_dt = {torch.float32: _lib.QSA_F32, torch.bfloat16: _lib.QSA_BF16}.get(q.dtype)
    if q_dt is None:
        raise TypeError("q must be float32 or bfloat16")
    _need(cu_q, torch.int32, "cu_q")
    _need(ctx_lens, torch.int32, "ctx_lens")
    _need(q_idx, torch.int8, "q_idx")
    _need(k_chunk, torch.int8, "k_chunk")
    _need(sel, torch.int32, "sel")
    _need(o, torch.float32, "o")
    _need(lse, torch.float32, "lse")
    B = ctx_lens.shape[0]
    d = cache.ring.shape[-1]
    if cu_q.shape[0] != B + 1 or q_idx.shape != (Nq, d) or k_chunk.shape != (Nq, d):
        raise ValueError("cu_q [B+1], q_idx and k_chunk [Nq, d] expected")
    if sel.shape != (Nq, topk) or o.shape != (Nq, Hq, D) or lse.shape != (Nq, Hq):
        raise ValueError("sel [Nq, topk], o [Nq, Hq, D] and lse [Nq, Hq] expected")
    s = cache.struct()
    _check(_lib.load().qsa_sparse_prefill(ctypes.byref(s), B, Nq, int(max_q_per_req), _ptr(cu_q),
                                          _ptr(ctx_lens), _ptr(q_idx), _ptr(k_chunk), _ptr(q),
                                          q_dt, Hq, int(max_blocks), int(topk), float(sm_scale),
                                          _ptr(sel), _ptr(o), _ptr(lse), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(),
                                          _stream(stream)), "qsa_sparse_prefill")


class QSASession:
    """Decode steps from host buffers to host buffers (qsa_session_*): the
    library owns the device buffers and overlaps each step's uploads and
    downloads with the kernels of its neighbours.  Host tensors should be
    pinned; they must stay unchanged (inputs) and untouched (outputs) until
    synchronize() returns."""

    def __init__(self, cache: QSACache, B: int, T: int, Hq: int, topk: int, num_splits: int,
                 max_blocks: int, max_new_tokens: int, sm_scale: float,
                 q_dtype=torch.bfloat16, stream=None):
        self.cache = cache  # keeps the caches alive
        self._struct = cache.struct()
        self.B, self.T, self.Hq, self.topk = B, T, Hq, topk
        self.D = cache.k_cache.shape[-1]
        self.d = cache.ring.shape[-1]
        self.q_dtype = q_dtype
        qd = {torch.float32: _lib.QSA_F32, torch.bfloat16: _lib.QSA_BF16}[q_dtype]
        lib = _lib.load()
        h = ctypes.c_void_p()
        cs = stream.cuda_stream if stream is not None else None
        _check(lib.qsa_session_create(ctypes.byref(self._struct), B, T, Hq, qd, topk, num_splits,
                                      max_blocks, max_new_tokens, float(sm_scale), cs,
                                      ctypes.byref(h)), "qsa_session_create")
        self._h = h

    def step(self, pos0, cu_new, k_new, q_idx, q, ctx_lens, n_sel, o, lse) -> None:
        B, T, Hq, D, d = self.B, self.T, self.Hq, self.D, self.d
        want = [(pos0, torch.int32, (B,)), (cu_new, torch.int32, (B + 1,)),
                (q_idx, torch.int8, (B, d)), (q, self.q_dtype, (B, T, Hq, D)),
                (ctx_lens, torch.int32, (B,)), (o, torch.float32, (B, T, Hq, D)),
                (lse, torch.float32, (B, T, Hq))]
        if n_sel is not None:
            want.append((n_sel, torch.int32, (B,)))
        for t, dt, shape in want:
            if t.is_cuda or t.dtype != dt or tuple(t.shape) != shape or not t.is_contiguous():
                raise ValueError(f"host tensor of dtype {dt} and shape {shape} expected")
        if (k_new.is_cuda or k_new.dtype != torch.int8 or k_new.dim() != 2 or
                k_new.shape[1] != d or not k_new.is_contiguous()):
            raise ValueError("k_new must be a contiguous host int8 tensor [N, d]")
        p = lambda t: None if t is None else t.data_ptr()
        _check(_lib.load().qsa_session_step_host(self._h, p(pos0), p(cu_new), p(k_new), p(q_idx),
                                                 p(q), p(ctx_lens), p(n_sel), p(o), p(lse)),
               "qsa_session_step_host")

    def streams(self) -> tuple[int, int, int]:
        """(upload, compute, download) stream handles."""
        a, b, c = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
        _check(_lib.load().qsa_session_streams(self._h, ctypes.byref(a), ctypes.byref(b),
                                               ctypes.byref(c)), "qsa_session_streams")
        return a.value or 0, b.value or 0, c.value or 0

    def synchronize(self) -> None:
        _check(_lib.load().qsa_session_synchronize(self._h), "qsa_session_synchronize")

    def close(self) -> None:
        if getattr(self, "_h", None):
            _lib.load().qsa_session_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def qsa_get_device_error(stream=None) -> tuple[int, int]:
    """Synchronises the stream; returns (status, flag bits) and clears the
    device error word."""
    lib = _lib.load()
    flags = ctypes.c_uint32(0)
    st = lib.qsa_get_device_error(_stream(stream), ctypes.byref(flags))
    return int(st), int(flags.value)
