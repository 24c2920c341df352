"""Multi-step MTP drafting with one indexer run (QSADraftDecode) against
the oracle.

The selecting step picks blocks for its query token at p0 from the
compressed keys of [0, p0]; draft steps k = 1..3 append their keys and
attend the kept blocks' tokens up to p0 + k plus every token after p0.  The
oracle side is built from its own pieces: selection over the step-0 prefix,
the token rows of that selection, token_set of query row k of an MTP query
with T = k + 1, attention per split and the LSE merge."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import qsa_harness as H
from oracle import qsa_ref as ref
from sparse_attention_decode_compress_b200 import QSADraftDecode
from workloads.qsa_inputs import WORKLOADS, make_batch, request_pages

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda_and_cleanup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _oracle_rows(b, r, L0, S, budget):
    """Oracle of the selecting step and its draft steps for request r."""
    w = b.w
    a = int(b.cu_ctx_host[r])
    k_all = b.k_idx[a:a + L0 + 3].cpu().numpy()
    kc0 = ref.compress_keys(k_all[:L0])
    scores = ref.block_scores(b.q_idx[r].cpu().numpy(), kc0, ref.selection_width(L0, 1))
    sel = ref.select_blocks(scores, budget // 4)
    tokens = ref.selection_tokens(sel, L0, 1, budget)
    # K / V of the whole final context, de-paged
    Lf = L0 + 3
    pages = request_pages(b, r)
    kst, kind = H._bits(b.k_cache[pages.to(b.device)].cpu())
    vst, _ = H._bits(b.v_cache[pages.to(b.device)].cpu())
    local = np.arange(pages.shape[0])
    ks = vs = None
    if b.k_scale is not None:
        tok_page = pages.numpy()[np.arange(Lf) // w.page_size]
        ks = b.k_scale.cpu().numpy()[tok_page]
        vs = b.v_scale.cpu().numpy()[tok_page]
    K = ref.StoredRows(ref.depage(kst, local, Lf, w.page_size), kind, ks)
    V = ref.StoredRows(ref.depage(vst, local, Lf, w.page_size), kind, vs)
    qb, qkind = H._bits(b.q[r].cpu())
    q = ref.decode_values(qb, qkind)                     # [4, Hq, D]: steps 0..3
    sm = 1.0 / np.sqrt(w.D)
    outs = []
    for k in range(4):
        toks = ref.token_set(sel, L0 + k, k + 1, k)
        op, lp = ref.split_attention(q[k], K, V, toks, sm, L0 + k, w.page_size, S)
        outs.append(ref.lse_merge(op, lp))
    return sel, tokens, outs, ref.compress_keys(k_all)


@pytest.mark.parametrize("name,lens,S,budget", [("mtp_verify", [16384 + 3, 9001, 6002, 2050], 2, 2048),
                                                ("mixed_fp8", [4099, 12345], 4, 2048),
                                                ("mtp_verify", [30001, 5003], 3, 512)])
def test_draft_steps_reuse_the_step0_selection(name, lens, S, budget):
    b = make_batch(replace(WORKLOADS[name], T=4), "cuda", ctx_lens=lens, seed=51)  # lengths L0 + 3
    w = b.w
    B = w.batch
    cache = H.build_cache(b)
    H.prefill(cache, b, 4)                                # positions [0, L0 - 1)
    L0 = (b.ctx_lens_host - 3).to(torch.int32)
    ends = b.cu_ctx_host[1:] - 3                          # row of position L0 - 1 in k_idx
    drv = QSADraftDecode(cache, B, w.Hq, budget, S, H.max_blocks_of(b))
    got = []
    for k in range(4):
        rows = (ends - 1 + k).to(b.device)
        k_new = b.k_idx[rows].contiguous()
        pos = (L0 - 1 + k).to(b.device)
        lens_k = (L0 + k).to(b.device)
        q = b.q[:, :k + 1].contiguous()
        if k == 0:
            tok, o, lse = drv.select(pos, k_new, b.q_idx, q, lens_k)
        else:
            tok, o, lse = drv.draft(pos, k_new, q, lens_k)
        st, flags = H.qsa_get_device_error()
        assert st == 0, (k, st, flags)
        got.append((o.cpu().numpy(), lse.cpu().numpy()))
    tok = tok.cpu().numpy()
    sel = drv.sel.cpu().numpy()
    for r in range(B):
        want_sel, want_tok, outs, kc_all = _oracle_rows(b, r, int(L0[r]), S, budget)
        assert np.array_equal(sel[r], want_sel), r
        assert np.array_equal(tok[r], want_tok), r        # the reused buffer, bit for bit
        for k in range(4):
            ma, rl = H.attn_errors(got[k][0][r], outs[k][0])
            le = H.lse_error(got[k][1][r], outs[k][1])
            assert ma <= H.MAX_ABS and rl <= H.REL_L2 and le <= H.LSE_ABS, (r, k, ma, rl, le)
        # the drafts' keys went to the side caches
        kc = H.gpu_kc_logical(b, cache, r)
        assert np.array_equal(kc.astype(np.int64), kc_all), r
    with pytest.raises(RuntimeError):
        drv.draft(pos, k_new, b.q.contiguous(), lens_k)   # a fourth draft has no reuse left
