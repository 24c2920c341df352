"""Test harness: runs the CUDA path (through the C ABI) and the CPU oracle on
the same seeded inputs and compares them.  Only tests import this module."""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle import qsa_ref as ref
from sparse_attention_decode_compress_b200 import (QSACache, QSADecodeStep, qsa_compress_append,
                                                   qsa_get_device_error)
from workloads.qsa_inputs import QSABatch, request_pages

# Tolerances of the attention outputs against the float64 oracle (fp32
# accumulation of bf16 / fp8 / fp32 inputs).
MAX_ABS = 1e-2
REL_L2 = 2e-3
LSE_ABS = 1e-4


def build_cache(batch: QSABatch) -> QSACache:
    w = batch.w
    return QSACache.allocate(batch.k_cache, batch.v_cache, batch.block_table, w.d_idx,
                             ring_rows=w.batch, k_scale=batch.k_scale, v_scale=batch.v_scale)


def prefill(cache: QSACache, batch: QSABatch, upto_minus: int) -> None:
    """Bulk-appends positions [0, L - upto_minus) of every request."""
    L = batch.ctx_lens_host
    n = (L - upto_minus).clamp(min=0)
    B = L.shape[0]
    if int(n.max()) == 0:
        return
    parts = [batch.k_idx[int(batch.cu_ctx_host[r]): int(batch.cu_ctx_host[r]) + int(n[r])]
             for r in range(B)]
    k_new = torch.cat(parts).contiguous()
    cu = torch.zeros(B + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(n, 0).to(torch.int32)
    pos0 = torch.zeros(B, dtype=torch.int32)
    dev = batch.device
    qsa_compress_append(cache, pos0.to(dev), cu.to(dev), k_new, int(n.max()))
    del k_new


def step_inputs(batch: QSABatch):
    """Inputs of one decode step: the last T tokens of every request."""
    w = batch.w
    T = w.T
    L = batch.ctx_lens_host
    B = L.shape[0]
    rows = torch.cat([torch.arange(int(batch.cu_ctx_host[r + 1]) - T, int(batch.cu_ctx_host[r + 1]))
                      for r in range(B)]).to(batch.device)
    k_new = batch.k_idx[rows].contiguous()
    cu = torch.arange(0, B * T + 1, T, dtype=torch.int32, device=batch.device)
    pos0 = (L - T).to(torch.int32).to(batch.device)
    n_sel = None
    if T > 1:
        n_sel = ((L - T) // 4 + 1).to(torch.int32).to(batch.device)
    return pos0, cu, k_new, n_sel


def max_blocks_of(batch: QSABatch) -> int:
    return int((batch.ctx_lens_host.max() + 3) // 4)


def run_gpu(batch: QSABatch, num_splits: int, keep_scores: bool = True, cache=None,
            check_errors: bool = True):
    """Prefill + one decode step on the GPU.  Returns the step object (its
    buffers hold sel, scores, o_part, lse_part, o, lse) and the cache."""
    w = batch.w
    if cache is None:
        cache = build_cache(batch)
        prefill(cache, batch, w.T)
    step = QSADecodeStep(cache, w.batch, w.T, w.Hq, w.topk, num_splits, max_blocks_of(batch),
                         keep_scores=keep_scores)
    pos0, cu, k_new, n_sel = step_inputs(batch)
    step(pos0, cu, k_new, batch.q_idx, batch.q, batch.ctx_lens, n_sel)
    if check_errors:
        st, flags = qsa_get_device_error()
        assert st == 0, f"device error status {st} flags {flags}"
    torch.cuda.synchronize()
    return step, cache


def _bits(t: torch.Tensor) -> tuple[np.ndarray, str]:
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16), "bf16"
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy(), "e4m3"
    return t.float().numpy(), "f32"


def oracle_request(batch: QSABatch, r: int, num_splits: int) -> dict:
    """The oracle's whole decode path for request r, from the logical inputs
    (host de-paging through the block table)."""
    w = batch.w
    L = int(batch.ctx_lens_host[r])
    a, e = int(batch.cu_ctx_host[r]), int(batch.cu_ctx_host[r + 1])
    k_idx = batch.k_idx[a:e].cpu().numpy()
    pages = request_pages(batch, r)
    pg_dev = pages.to(batch.device)
    kst, kind = _bits(batch.k_cache[pg_dev].cpu())
    vst, _ = _bits(batch.v_cache[pg_dev].cpu())
    local = np.arange(pages.shape[0])
    Kst = ref.depage(kst, local, L, w.page_size)
    Vst = ref.depage(vst, local, L, w.page_size)
    ks = vs = None
    if batch.k_scale is not None:
        tok_page = pages.numpy()[np.arange(L) // w.page_size]
        ks = batch.k_scale.cpu().numpy()[tok_page]
        vs = batch.v_scale.cpu().numpy()[tok_page]
    K = ref.StoredRows(Kst, kind, ks)
    V = ref.StoredRows(Vst, kind, vs)
    qb, qkind = _bits(batch.q[r].cpu())
    q = ref.decode_values(qb, qkind)
    out = ref.decode_request(k_idx, batch.q_idx[r].cpu().numpy(), q, K, V, w.T, w.page_size,
                             num_splits, w.topk)
    out["L"] = L
    return out


def unpack_kc_pages(pages: np.ndarray, P: int, d: int) -> np.ndarray:
    """Compressed-key values [n, P/4, d] (int64) of packed pages [n, bytes],
    read by the layout include/qsa.h states at qsa_kc_page_bytes: R = P/4
    rows of d low bytes, then 32-bit field words, word w*R + row holding
    dims 16w..16w+15 of the row, dim 16w+4s+k at bits 8k+2s; value =
    256*(field-2)+low."""
    R = P // 4
    n = pages.shape[0]
    lo = pages[:, :R * d].reshape(n, R, d).astype(np.int64)
    hib = pages[:, R * d:R * d + R * d // 4].reshape(n, d // 16, R, 4).transpose(0, 2, 1, 3)
    hib = hib.astype(np.int64)
    s = np.arange(4)
    f = (hib[:, :, :, None, :] >> (2 * s)[:, None]) & 3   # [n, R, w, s, k]
    return 256 * (f.reshape(n, R, d) - 2) + lo


def gpu_kc_logical(batch: QSABatch, cache: QSACache, r: int) -> np.ndarray:
    L = int(batch.ctx_lens_host[r])
    pages = request_pages(batch, r)
    kcp = unpack_kc_pages(cache.kc[pages.to(batch.device)].cpu().numpy(), batch.w.page_size,
                          batch.w.d_idx)
    return ref.depage_kc(kcp, np.arange(pages.shape[0]), L, batch.w.page_size)


def attn_errors(got: np.ndarray, want: np.ndarray) -> tuple[float, float]:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    max_abs = float(np.max(np.abs(got - want))) if got.size else 0.0
    den = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(got - want) / den) if den > 0 else float(np.linalg.norm(got - want))
    return max_abs, rel


def lse_error(got: np.ndarray, want: np.ndarray) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    inf_g, inf_w = np.isneginf(got), np.isneginf(want)
    assert np.array_equal(inf_g, inf_w), "empty (-inf) rows differ"
    fin = ~inf_w
    return float(np.max(np.abs(got[fin] - want[fin]))) if fin.any() else 0.0


def check_request(batch: QSABatch, step: QSADecodeStep, cache: QSACache, r: int,
                  num_splits: int, check_kc: bool = True) -> dict:
    """Element-wise comparison of one request against the oracle."""
    w = batch.w
    want = oracle_request(batch, r, num_splits)
    L = want["L"]
    n_sel = ref.selection_width(L, w.T)
    if check_kc:
        kc = gpu_kc_logical(batch, cache, r)
        assert np.array_equal(kc.astype(np.int64), want["kc"]), f"kc mismatch r={r}"
        # ring: newest positions of the request
        ring = cache.ring[r].cpu().numpy()
        a = int(batch.cu_ctx_host[r])
        kid = batch.k_idx[a + max(0, L - 4): a + L].cpu().numpy()
        for j, p in enumerate(range(max(0, L - 4), L)):
            assert np.array_equal(ring[p % 4], kid[j]), f"ring slot mismatch r={r} p={p}"
    if step.scores is not None:
        sc = step.scores[r, :n_sel].cpu().numpy().astype(np.int64)
        assert np.array_equal(sc, want["scores"]), f"score mismatch r={r}"
    sel = step.sel[r].cpu().numpy()
    assert np.array_equal(sel, want["sel"]), f"selection mismatch r={r}"
    o_part = step.o_part[:, r].cpu().numpy()
    lse_part = step.lse_part[:, r].cpu().numpy()
    ma, rl = attn_errors(o_part, want["o_part"])
    le = lse_error(lse_part, want["lse_part"])
    assert ma <= MAX_ABS and rl <= REL_L2, f"o_part r={r}: max_abs {ma:.3e} rel_l2 {rl:.3e}"
    assert le <= LSE_ABS, f"lse_part r={r}: {le:.3e}"
    o = step.o[r].cpu().numpy()
    lse = step.lse[r].cpu().numpy()
    ma2, rl2 = attn_errors(o, want["o"])
    le2 = lse_error(lse, want["lse"])
    assert ma2 <= MAX_ABS and rl2 <= REL_L2, f"merged o r={r}: max_abs {ma2:.3e} rel_l2 {rl2:.3e}"
    assert le2 <= LSE_ABS, f"merged lse r={r}: {le2:.3e}"
    return dict(max_abs=max(ma, ma2), rel_l2=max(rl, rl2), lse=max(le, le2))


def check_properties(batch: QSABatch, step: QSADecodeStep) -> None:
    """Properties of every request that hold at any size."""
    w = batch.w
    sel = step.sel.cpu()
    L = batch.ctx_lens_host
    n_sel = (L - w.T) // 4 + 1
    valid = sel >= 0
    cnt = valid.sum(dim=1)
    assert torch.equal(cnt, torch.minimum(n_sel, torch.tensor(w.topk))), "kept count"
    # valid prefix, then -1
    assert torch.equal(valid, torch.arange(w.topk)[None, :] < cnt[:, None]), "padding layout"
    d = sel[:, 1:] - sel[:, :-1]
    both = valid[:, 1:] & valid[:, :-1]
    assert bool((d[both] > 0).all()), "selection not strictly ascending"
    assert bool((sel[valid] < n_sel.repeat_interleave(cnt)).all()), "selected block out of range"
    if batch.planted_host is not None:
        for r in range(w.batch):
            pl = [b for b in batch.planted_host[r].tolist() if b >= 0]
            assert set(pl) <= set(sel[r].tolist()), f"planted r={r}"
    o = step.o.cpu()
    assert bool(torch.isfinite(o).all()) and bool(torch.isfinite(step.lse.cpu()).all())


def check_index_every_request(batch: QSABatch, sel: torch.Tensor, scores: torch.Tensor | None,
                              topk: int | None = None, workers: int = 16) -> int:
    """Bit-exact comparison of the selection rows (and, when given, the
    scores) of EVERY request with the oracle's indexer path, run request by
    request in a pool of spawn worker processes.  The raw keys go to the
    workers one request at a time, with a bounded number in flight, so host
    memory stays bounded at any batch size.  Returns the requests checked."""
    import oracle_index
    w = batch.w
    topk = w.topk if topk is None else topk
    sel_h = sel.cpu().numpy()
    sc_dev = scores
    pending = {}
    checked = 0

    def settle(fut, r):
        nonlocal checked
        want_sc, want_sel = fut.result()
        assert np.array_equal(sel_h[r], want_sel), f"selection mismatch r={r}"
        if sc_dev is not None:
            got = sc_dev[r, :want_sc.shape[0]].cpu().numpy().astype(np.int64)
            assert np.array_equal(got, want_sc), f"score mismatch r={r}"
        checked += 1

    n_workers = oracle_index.pool_size(workers)
    with oracle_index.pool(n_workers) as ex:
        limit = 2 * n_workers
        for r in range(w.batch):
            a, e = int(batch.cu_ctx_host[r]), int(batch.cu_ctx_host[r + 1])
            k = batch.k_idx[a:e].cpu().numpy()
            q = batch.q_idx[r].cpu().numpy()
            pending[ex.submit(oracle_index.index_request, k, q, w.T, topk)] = r
            if len(pending) >= limit:
                fut = next(iter(pending))
                settle(fut, pending.pop(fut))
        for fut, r in list(pending.items()):
            settle(fut, r)
    return checked


def sample_requests(L: torch.Tensor, k: int = 16) -> list[int]:
    """k requests spread over the context-length order (shortest and longest
    included)."""
    order = torch.argsort(L).tolist()
    n = len(order)
    if n <= k:
        return sorted(order)
    pick = {order[round(i * (n - 1) / (k - 1))] for i in range(k)}
    return sorted(pick)
