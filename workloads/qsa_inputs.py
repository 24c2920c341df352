"""Seeded synthetic inputs for decode-time QSA workloads.

This module only draws random numbers and lays them out; it holds none of
the method's arithmetic (no compression, scoring, selection or attention).
Both the CUDA path (through ``bench.py`` and the GPU tests) and the CPU
oracle (through the tests) take their inputs from here.

The five named workloads follow the long-context serving setting of the
source pages (262,144-token contexts, "extendable to 1,000,000"; GQA query
heads over few KV heads; a 4-token micro-block indexer keeping 512 blocks).
The pages' own workload (a serving trace) is not available, so these seeded
distributions stand in for it:

* K/V/Q ~ N(0, 1), stored as float32, bfloat16 or FP8 E4M3 with one float32
  scale per (page, kv head) equal to amax / 448 (round-to-nearest-even);
* raw indexer keys and the indexer query ~ uniform integers in [-127, 127];
* optional planted spans: 8 distinct, block-aligned 4-token spans per request
  whose indexer keys equal the request's indexer query (so they score
  highest, tied with each other) and whose attention keys, per kv head g,
  are alpha * mean of the query heads of g, alpha = 8 * G / sqrt(D) (scaled
  logit about 8, so the softmax is sharply peaked on them);
* paged caches with a random permutation of physical pages (identity for
  the tiny workload) and a block table padded with -1.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

RATIO = 4


@dataclass(frozen=True)
class QSAWorkload:
    name: str
    batch: int
    ctx: str                 # "fixed:<L>", "uniform:<lo>:<hi>", "loguniform:<lo>:<hi>"
    T: int                   # query tokens per request (1, or 4 for MTP verify)
    Hq: int
    Hkv: int
    D: int
    d_idx: int
    kv_dtype: str            # 'f32' | 'bf16' | 'e4m3'
    q_dtype: str             # 'f32' | 'bf16'
    page_size: int
    topk: int = 512
    splits: tuple = (1,)
    random_table: bool = True
    planted: int = 0
    seed: int = 0
    description: str = ""


WORKLOADS = {
    "tiny": QSAWorkload(
        "tiny", 1, "fixed:4096", 1, 8, 1, 64, 32, "f32", "f32", 16, 512, (1,),
        random_table=False, planted=0, seed=0,
        description="batch 1, context 4096, 8 q / 1 kv heads, D 64, fp32; indexer d 32; "
                    "page 16, identity block table; 1 KV split"),
    "b32_32k": QSAWorkload(
        "b32_32k", 32, "fixed:32768", 1, 16, 2, 128, 128, "bf16", "bf16", 64, 512, (2,),
        planted=8, description="batch 32 x 32768 ctx, GQA 16/2, D 128, bf16, 8 planted spans, "
                               "page 64 random table, 2 KV splits"),
    "b128_256k": QSAWorkload(
        "b128_256k", 128, "fixed:262144", 1, 16, 2, 128, 128, "bf16", "bf16", 64, 512, (1, 2, 4),
        planted=8, description="batch 128 x 262144 ctx, GQA 16/2, D 128, bf16, planted spans, "
                               "page 64 random table, 1/2/4 KV splits"),
    "mtp_verify": QSAWorkload(
        "mtp_verify", 64, "uniform:16384:262144", 4, 16, 2, 128, 128, "bf16", "bf16", 64, 512,
        (2,), planted=8, description="batch 64, ctx ~U[16384, 262144], 4 query tokens (1 + 3 "
                                     "speculative, causal), GQA 16/2, bf16, 2 KV splits"),
    "mixed_fp8": QSAWorkload(
        "mixed_fp8", 256, "loguniform:4096:1048576", 1, 32, 4, 128, 128, "e4m3", "bf16", 64, 512,
        (4,), planted=0, description="batch 256, ctx log-uniform [4096, 1048576], GQA 32/4, "
                                     "K/V fp8 E4M3 + fp32 scale per (page, kv head), Q bf16, "
                                     "4 KV splits"),
}

TORCH_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.float8_e4m3fn}


def draw_ctx_lens(w: QSAWorkload, gen: torch.Generator) -> torch.Tensor:
    """Context lengths (tokens, including the new query tokens), int64 [B]."""
    kind, *args = w.ctx.split(":")
    if kind == "fixed":
        return torch.full((w.batch,), int(args[0]), dtype=torch.int64)
    lo, hi = int(args[0]), int(args[1])
    if kind == "uniform":
        return torch.randint(lo, hi + 1, (w.batch,), generator=gen, dtype=torch.int64)
    if kind == "loguniform":
        u = torch.rand(w.batch, generator=gen, dtype=torch.float64)
        L = torch.floor(torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo))))
        return L.clamp_(lo, hi).to(torch.int64)
    raise ValueError(w.ctx)


@dataclass
class QSABatch:
    """All inputs of one batch.  Device tensors live on ``device``; the small
    metadata tensors also have host copies (``*_host``)."""
    w: QSAWorkload
    device: torch.device
    ctx_lens_host: torch.Tensor          # int64 [B]
    block_table_host: torch.Tensor       # int32 [B, max_pages], -1 padded
    num_pages: int
    ctx_lens: torch.Tensor               # int32 [B] on device
    block_table: torch.Tensor            # int32 [B, max_pages] on device
    k_cache: torch.Tensor                # [num_pages, P, Hkv, D]
    v_cache: torch.Tensor
    k_scale: torch.Tensor | None         # float32 [num_pages, Hkv] (fp8 only)
    v_scale: torch.Tensor | None
    q: torch.Tensor                      # [B, T, Hq, D]
    q_idx: torch.Tensor                  # int8 [B, d]
    k_idx: torch.Tensor                  # int8 [sum L, d], logical token order
    cu_ctx_host: torch.Tensor            # int64 [B+1] offsets of requests in k_idx
    planted_host: torch.Tensor | None    # int64 [B, planted] block indices
    extra: dict = field(default_factory=dict)


def make_batch(w: QSAWorkload, device="cpu", seed: int | None = None,
               ctx_lens: list[int] | None = None, batch: int | None = None) -> QSABatch:
    """Draw one batch of workload ``w`` on ``device``.

    ``batch`` / ``ctx_lens`` override the workload's batch size and context
    lengths (used for edge cases and for sampled CPU runs)."""
    device = torch.device(device)
    seed = w.seed if seed is None else seed
    if ctx_lens is not None:
        w = replace(w, batch=len(ctx_lens))
    elif batch is not None:
        w = replace(w, batch=batch)
    B, P = w.batch, w.page_size
    meta = torch.Generator().manual_seed(seed)
    if ctx_lens is None:
        L = draw_ctx_lens(w, meta)
    else:
        L = torch.tensor(ctx_lens, dtype=torch.int64)
    if int(L.min()) < w.T:
        raise ValueError("every context must hold at least the T query tokens")
    pages_per = (L + P - 1) // P
    num_pages = int(pages_per.sum())
    max_pages = int(pages_per.max())
    phys = torch.randperm(num_pages, generator=meta) if w.random_table else torch.arange(num_pages)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    off = 0
    for r in range(B):
        n = int(pages_per[r])
        table[r, :n] = phys[off:off + n].to(torch.int32)
        off += n

    planted = None
    if w.planted:
        # requests too short to hold the spans get none (row of -1)
        planted = torch.full((B, w.planted), -1, dtype=torch.int64)
        for r in range(B):
            nfull = (int(L[r]) - w.T + 1) // RATIO        # complete blocks within [0, p0]
            if nfull >= w.planted:
                planted[r] = torch.randperm(nfull, generator=meta)[:w.planted]

    dev_gen = torch.Generator(device=device).manual_seed(seed + 1)
    qdt = TORCH_DTYPES[w.q_dtype]
    q = torch.randn((B, w.T, w.Hq, w.D), generator=dev_gen, device=device,
                    dtype=torch.float32).to(qdt)
    q_idx = torch.randint(-127, 128, (B, w.d_idx), generator=dev_gen, device=device,
                          dtype=torch.int8)
    cu = torch.zeros(B + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(L, 0)
    k_idx = torch.randint(-127, 128, (int(cu[-1]), w.d_idx), generator=dev_gen,
                          device=device, dtype=torch.int8)

    G = w.Hq // w.Hkv
    alpha = 8.0 * G / math.sqrt(w.D)
    shape = (num_pages, P, w.Hkv, w.D)
    k_scale = v_scale = None
    table_dev = table.to(device)

    # planted positions -> (physical page, offset) and the planted key values
    plant_pages = plant_offs = plant_rows = plant_k = None
    if planted is not None and bool((planted >= 0).any()):
        toks = (planted[:, :, None] * RATIO + torch.arange(RATIO)[None, None, :]).reshape(B, -1)
        rows = torch.arange(B)[:, None].expand_as(toks)
        keep = (toks >= 0).reshape(-1)
        toks_k = toks.reshape(-1)[keep]
        rows_k = rows.reshape(-1)[keep]
        plant_pages = table[rows_k, toks_k // P].to(torch.int64)
        plant_offs = toks_k % P
        plant_rows = rows_k
        qm = q[:, 0].float().reshape(B, w.Hkv, G, w.D).mean(dim=2) * alpha   # [B, Hkv, D]
        plant_k = qm.cpu()[plant_rows]                                      # [n, Hkv, D]
        # indexer keys of planted tokens = the request's indexer query
        glob = (cu[:-1][rows_k] + toks_k).to(device)
        k_idx[glob] = q_idx[plant_rows.to(device)]

    if w.kv_dtype in ("f32", "bf16"):
        dt = TORCH_DTYPES[w.kv_dtype]
        k_cache = torch.randn(shape, generator=dev_gen, device=device, dtype=torch.float32).to(dt) \
            if dt == torch.float32 else _randn_bf16(shape, dev_gen, device)
        v_cache = torch.randn(shape, generator=dev_gen, device=device, dtype=torch.float32).to(dt) \
            if dt == torch.float32 else _randn_bf16(shape, dev_gen, device)
        if plant_pages is not None:
            k_cache[plant_pages.to(device), plant_offs.to(device)] = plant_k.to(device=device, dtype=dt)
    else:
        k_cache = torch.empty(shape, device=device, dtype=torch.float8_e4m3fn)
        v_cache = torch.empty(shape, device=device, dtype=torch.float8_e4m3fn)
        k_scale = torch.empty((num_pages, w.Hkv), device=device, dtype=torch.float32)
        v_scale = torch.empty((num_pages, w.Hkv), device=device, dtype=torch.float32)
        chunk = max(1, (1 << 28) // (P * w.Hkv * w.D))      # ~1 GiB of float32 per chunk
        for p0 in range(0, num_pages, chunk):
            p1 = min(num_pages, p0 + chunk)
            for cache, scale in ((k_cache, k_scale), (v_cache, v_scale)):
                x = torch.randn((p1 - p0, P, w.Hkv, w.D), generator=dev_gen, device=device,
                                dtype=torch.float32)
                if cache is k_cache and plant_pages is not None:
                    sel = (plant_pages >= p0) & (plant_pages < p1)
                    if bool(sel.any()):
                        x[(plant_pages[sel] - p0).to(device), plant_offs[sel].to(device)] = \
                            plant_k[sel].to(device)
                amax = x.abs().amax(dim=(1, 3))                       # [pages, Hkv]
                s = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
                cache[p0:p1] = (x / s[:, None, :, None]).to(torch.float8_e4m3fn)
                scale[p0:p1] = s
                del x

    return QSABatch(w=w, device=device, ctx_lens_host=L, block_table_host=table,
                    num_pages=num_pages, ctx_lens=L.to(torch.int32).to(device),
                    block_table=table_dev, k_cache=k_cache, v_cache=v_cache,
                    k_scale=k_scale, v_scale=v_scale, q=q, q_idx=q_idx, k_idx=k_idx,
                    cu_ctx_host=cu, planted_host=planted)


def _randn_bf16(shape, gen, device):
    """N(0,1) bf16 tensor drawn in slabs (bounded float32 temporaries)."""
    out = torch.empty(shape, device=device, dtype=torch.bfloat16)
    flat = out.view(-1)
    step = 1 << 28
    for a in range(0, flat.numel(), step):
        b = min(flat.numel(), a + step)
        flat[a:b] = torch.randn(b - a, generator=gen, device=device, dtype=torch.float32)
    return out


def request_pages(batch: QSABatch, r: int) -> torch.Tensor:
    """Physical pages of request r in logical order (int64, host)."""
    L = int(batch.ctx_lens_host[r])
    n = (L + batch.w.page_size - 1) // batch.w.page_size
    return batch.block_table_host[r, :n].to(torch.int64)


def norm_indexer_inputs(batch: QSABatch, seed: int = 0, weight_std: float = 0.0) -> dict:
    """Inputs of the normalised-pooling indexer variant for `batch`: raw
    indexer keys k [sum L, d] and queries q [B, d], bfloat16 ~ N(0, 1); the
    planted spans' keys (if any) equal their request's query; an optional
    per-dim norm weight w ~ N(0, weight_std^2) (float32 [d], None for 0)."""
    w = batch.w
    device = batch.device
    gen = torch.Generator(device=device).manual_seed(seed + 7)
    n_tok = int(batch.cu_ctx_host[-1])
    k = torch.randn((n_tok, w.d_idx), generator=gen, device=device,
                    dtype=torch.float32).to(torch.bfloat16)
    q = torch.randn((w.batch, w.d_idx), generator=gen, device=device,
                    dtype=torch.float32).to(torch.bfloat16)
    if batch.planted_host is not None:
        for r in range(w.batch):
            for b in batch.planted_host[r].tolist():
                if b >= 0:
                    a = int(batch.cu_ctx_host[r]) + RATIO * b
                    k[a:a + RATIO] = q[r]
    weight = None
    if weight_std > 0:
        weight = torch.randn(w.d_idx, generator=gen, device=device,
                             dtype=torch.float32) * weight_std
    return dict(k=k, q=q, weight=weight)


def prefill_inputs(batch: QSABatch, n_q: list[int], seed: int = 0) -> dict:
    """Inputs of a sparse prefill over `batch`: the newest n_q[r] tokens of
    request r are its query tokens.  Returns cu_q (int32 [B+1]), their rows
    in batch.k_idx (the chunk's raw indexer keys), per-token indexer queries
    q_idx (int8 [Nq, d], uniform in [-127, 127]) and attention queries q
    ([Nq, Hq, D] of the workload's query dtype, ~ N(0, 1))."""
    w = batch.w
    device = batch.device
    L = batch.ctx_lens_host
    if len(n_q) != w.batch or any(int(n) > int(l) or n < 0 for n, l in zip(n_q, L.tolist())):
        raise ValueError("one chunk length per request, at most its context")
    cu = torch.zeros(w.batch + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(torch.tensor(n_q, dtype=torch.int64), 0)
    rows = torch.cat([torch.arange(int(batch.cu_ctx_host[r + 1]) - n_q[r],
                                   int(batch.cu_ctx_host[r + 1])) for r in range(w.batch)])
    gen = torch.Generator(device=device).manual_seed(seed + 11)
    nq = int(cu[-1])
    q_idx = torch.randint(-127, 128, (nq, w.d_idx), generator=gen, device=device, dtype=torch.int8)
    q = torch.randn((nq, w.Hq, w.D), generator=gen, device=device,
                    dtype=torch.float32).to(TORCH_DTYPES[w.q_dtype])
    return dict(cu_q=cu.to(torch.int32), rows=rows, q_idx=q_idx, q=q,
                k_chunk=batch.k_idx[rows.to(device)].contiguous())
