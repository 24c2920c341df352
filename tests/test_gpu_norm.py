"""GPU parity of the normalised-pooling indexer variant (float compressed
keys and scores) against its oracle (oracle/qsa_ref_norm.py).

Float scores are compared within the bound the stored float16 keys allow,
atol = 2^-10 * |q|_2 * sqrt(d) * max|1 + w| (twice the bound of one float16
rounding per key element); the selection must be an admissible top-k of the
oracle's scores at that atol, and bit-exact as a top-k of the GPU's own
scores; attention on the kept set within the usual tolerances."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import qsa_harness as H
from oracle import qsa_ref as ref
from oracle import qsa_ref_norm as nref
from sparse_attention_decode_compress_b200 import api
from workloads.qsa_inputs import WORKLOADS, make_batch, norm_indexer_inputs, request_pages

pytestmark = pytest.mark.gpu

EPS = 1e-6


@pytest.fixture(autouse=True)
def _cuda_and_cleanup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _bf16_f64(t: torch.Tensor) -> np.ndarray:
    return ref.bf16_bits_to_f64(t.cpu().view(torch.int16).numpy().view(np.uint16))


def _run(b, ni, S, append_one_by_one=False):
    """Prefill and one decode step of the normalised indexer, then the sparse
    decode on its selection."""
    w = b.w
    cache = H.build_cache(b)
    kcn, ring = api.allocate_norm_caches(cache, w.batch)
    L = b.ctx_lens_host
    B = w.batch
    dev = b.device
    k = ni["k"]

    def append(lo, hi):   # positions [lo_r, hi_r) of every request
        n = (hi - lo).clamp(min=0)
        if int(n.max()) == 0:
            return
        rows = torch.cat([torch.arange(int(b.cu_ctx_host[r]) + int(lo[r]),
                                       int(b.cu_ctx_host[r]) + int(lo[r]) + int(n[r]))
                          for r in range(B)])
        cu = torch.zeros(B + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(n, 0).to(torch.int32)
        api.qsa_compress_append_norm(cache, kcn, ring, ni["weight"], EPS, lo.to(torch.int32).to(dev),
                                     cu.to(dev), k[rows.to(dev)].contiguous(), int(n.max()))

    zero = torch.zeros_like(L)
    if append_one_by_one:
        append(zero, L - 6)
        for j in range(6, 0, -1):
            append(L - j, L - j + 1)
    else:
        append(zero, L - w.T)
        append(L - w.T, L)
    max_blocks = H.max_blocks_of(b)
    n_sel = ((L - w.T) // 4 + 1).to(torch.int32).to(dev) if w.T > 1 else None
    sel = torch.empty((B, w.topk), dtype=torch.int32, device=dev)
    scores = torch.empty((B, max_blocks), dtype=torch.float32, device=dev)
    ws = api.new_workspace(api.qsa_index_topk_workspace_bytes(B, max_blocks), dev)
    api.qsa_index_topk_norm(cache, kcn, ni["q"], b.ctx_lens, n_sel, max_blocks, w.topk, sel,
                            scores, ws)
    D = b.k_cache.shape[-1]
    o_part = torch.empty((S, B, w.T, w.Hq, D), device=dev)
    lse_part = torch.empty((S, B, w.T, w.Hq), device=dev)
    o = torch.empty((B, w.T, w.Hq, D), device=dev)
    lse = torch.empty((B, w.T, w.Hq), device=dev)
    wsd = api.new_workspace(api.qsa_sparse_decode_workspace_bytes(B, w.T, w.Hq, b.k_cache.shape[2],
                                                                  D, w.topk, S), dev)
    api.qsa_sparse_decode_merged(cache, b.q, b.ctx_lens, sel, 1.0 / np.sqrt(D), S, o_part,
                                 lse_part, o, lse, wsd)
    st, flags = api.qsa_get_device_error()
    assert st == 0, (st, flags)
    torch.cuda.synchronize()
    return dict(cache=cache, kcn=kcn, ring=ring, sel=sel, scores=scores, o=o, lse=lse)


def _check(b, ni, got, S):
    w = b.w
    d = w.d_idx
    wt = None if ni["weight"] is None else ni["weight"].cpu().numpy().astype(np.float64)
    wmax = 1.0 if wt is None else float(np.max(np.abs(1.0 + wt)))
    k_all = _bf16_f64(ni["k"])
    q_all = _bf16_f64(ni["q"])
    sel_g = got["sel"].cpu().numpy()
    sc_g = got["scores"].cpu().numpy().astype(np.float64)
    kcn = got["kcn"].cpu().float().numpy().astype(np.float64)
    ring = got["ring"].cpu().view(torch.int16).numpy()
    k_bits = ni["k"].cpu().view(torch.int16).numpy()
    P = w.page_size
    for r in range(w.batch):
        L = int(b.ctx_lens_host[r])
        a = int(b.cu_ctx_host[r])
        kc_o = nref.compress_keys_norm(k_all[a:a + L], EPS, wt)
        # compressed keys: one float16 rounding of the exact value
        pages = request_pages(b, r).numpy()
        kc_g = ref.depage_kc(kcn[pages], np.arange(pages.shape[0]), L, P)
        assert np.all(np.abs(kc_g - kc_o) <= 2.0 ** -10 * np.abs(kc_o) + 2.0 ** -24), r
        # ring: the newest raw keys, bit for bit
        for p in range(max(0, L - 4), L):
            assert np.array_equal(ring[r, p % 4], k_bits[a + p]), (r, p)
        n_sel = ref.selection_width(L, w.T)
        s_o = nref.block_scores_f(q_all[r], kc_o, n_sel)
        atol = 2.0 ** -10 * float(np.linalg.norm(q_all[r])) * np.sqrt(d) * wmax
        assert np.max(np.abs(sc_g[r, :n_sel] - s_o)) <= atol, r
        assert nref.selection_within_tolerance(sel_g[r], s_o, w.topk, atol), r
        # the kernel's selection is exactly the top-k of its own scores
        assert np.array_equal(sel_g[r], nref.select_blocks_f(sc_g[r, :n_sel], w.topk)), r
        if b.planted_host is not None:
            pl = [x for x in b.planted_host[r].tolist() if x >= 0]
            assert set(pl) <= set(sel_g[r].tolist()), r
        # attention over the kept set against the oracle on that set
        want = _oracle_attention(b, r, sel_g[r], S)
        ma, rl = H.attn_errors(got["o"][r].cpu().numpy(), want[0])
        le = H.lse_error(got["lse"][r].cpu().numpy(), want[1])
        assert ma <= H.MAX_ABS and rl <= H.REL_L2 and le <= H.LSE_ABS, (r, ma, rl, le)


def _oracle_attention(b, r, sel, S):
    w = b.w
    L = int(b.ctx_lens_host[r])
    pages = request_pages(b, r)
    kst, kind = H._bits(b.k_cache[pages.to(b.device)].cpu())
    vst, _ = H._bits(b.v_cache[pages.to(b.device)].cpu())
    local = np.arange(pages.shape[0])
    ks = vs = None
    if b.k_scale is not None:
        tp = pages.numpy()[np.arange(L) // w.page_size]
        ks, vs = b.k_scale.cpu().numpy()[tp], b.v_scale.cpu().numpy()[tp]
    K = ref.StoredRows(ref.depage(kst, local, L, w.page_size), kind, ks)
    V = ref.StoredRows(ref.depage(vst, local, L, w.page_size), kind, vs)
    qb, qkind = H._bits(b.q[r].cpu())
    q = ref.decode_values(qb, qkind)
    o = np.zeros((w.T, w.Hq, w.D))
    lse = np.zeros((w.T, w.Hq))
    for t in range(w.T):
        toks = ref.token_set(sel, L, w.T, t)
        op, lp = ref.split_attention(q[t], K, V, toks, 1.0 / np.sqrt(w.D), L, w.page_size, S)
        o[t], lse[t] = ref.lse_merge(op, lp)
    return o, lse


@pytest.mark.parametrize("name,over,lens,S,wstd", [
    ("b32_32k", dict(), [32768, 9001, 4099, 2047], 2, 0.0),
    ("b32_32k", dict(), [20000, 13001], 2, 0.3),
    ("b32_32k", dict(d_idx=64, page_size=16), [12345, 6002], 3, 0.0),
    ("b32_32k", dict(d_idx=32, page_size=12), [9000, 4097], 2, 0.1),
    ("mtp_verify", dict(), [16384 + 3, 9001, 4100], 2, 0.0),
    ("mixed_fp8", dict(), [4096, 30007], 4, 0.0),
    ("b128_256k", dict(), [262144, 100003], 2, 0.0),
])
def test_norm_indexer_against_the_oracle(name, over, lens, S, wstd):
    w = replace(WORKLOADS[name], **over)
    b = make_batch(w, "cuda", ctx_lens=lens, seed=61)
    ni = norm_indexer_inputs(b, seed=61, weight_std=wstd)
    _check(b, ni, _run(b, ni, S), S)


def test_norm_indexer_one_token_appends():
    w = replace(WORKLOADS["b32_32k"], planted=0)
    b = make_batch(w, "cuda", ctx_lens=[3001, 4099, 2050], seed=62)
    ni = norm_indexer_inputs(b, seed=62, weight_std=0.2)
    _check(b, ni, _run(b, ni, 2, append_one_by_one=True), 2)


def test_norm_indexer_ties_take_the_lowest_blocks():
    """Equal raw keys give equal compressed keys and equal scores: the
    first topk blocks are kept (the exact fallback on float keys)."""
    w = replace(WORKLOADS["b32_32k"], planted=0)
    b = make_batch(w, "cuda", ctx_lens=[32768, 20000], seed=63)
    ni = norm_indexer_inputs(b, seed=63)
    ni["k"][:] = ni["k"][0].clone()
    got = _run(b, ni, 2)
    assert got["sel"][0].cpu().tolist() == list(range(512))
    assert got["sel"][1].cpu().tolist() == list(range(512))
    _check(b, ni, got, 2)


# More requests than SMs, each at most 32,768 blocks: the selection on float
# keys runs in CTAs of 512 threads, two per SM (its two passes, and the exact
# fallback when every score ties).
@pytest.mark.parametrize("ties", [False, True])
def test_norm_indexer_more_requests_than_sms(ties):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    lens = [32768, 20001] + [2100 + 61 * i for i in range(sms)]
    w = replace(WORKLOADS["b32_32k"], planted=0 if ties else 8)
    b = make_batch(w, "cuda", ctx_lens=lens, seed=64)
    ni = norm_indexer_inputs(b, seed=64)
    if ties:
        ni["k"][:] = ni["k"][0].clone()
    got = _run(b, ni, 2)
    if ties:
        for r in range(len(lens)):
            assert got["sel"][r].cpu().tolist() == list(range(512)), r
    _check(b, ni, got, 2)
