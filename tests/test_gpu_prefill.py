"""GPU parity of qsa_sparse_prefill (tensor-core scan of every query token
against its prefix, per-token selection and attention) against the prefill
oracle (oracle/qsa_ref_prefill.py): selected blocks bit for bit, attention
within max-abs 1e-2 / rel-L2 2e-3 and LSE within 1e-4, on every query token.

Chunks start at position 0 (a whole prefill, dense for the first 2,048
positions), mid-block (the first block holds tokens from before the chunk)
and deep in long contexts; indexer dims 128, 64 and 32 take the 128-, 64-
and 32-byte swizzled operand layouts of the tensor-core scan."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import qsa_harness as H
from oracle import qsa_ref as ref
from oracle import qsa_ref_prefill as pre
from sparse_attention_decode_compress_b200 import api
from workloads.qsa_inputs import WORKLOADS, make_batch, prefill_inputs, request_pages

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda_and_cleanup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def run_prefill(b, pi, topk):
    """Appends every request's keys (the chunk last), then one prefill call."""
    w = b.w
    cache = H.build_cache(b)
    H.prefill(cache, b, 0)                       # all cached tokens, chunk included
    Nq = int(pi["cu_q"][-1])
    n_q = (pi["cu_q"][1:] - pi["cu_q"][:-1])
    max_blocks = H.max_blocks_of(b)
    Hkv, D = b.k_cache.shape[2], b.k_cache.shape[3]
    sel = torch.full((Nq, topk), -7, dtype=torch.int32, device="cuda")
    o = torch.full((Nq, w.Hq, D), 7.0, device="cuda")
    lse = torch.full((Nq, w.Hq), 7.0, device="cuda")
    ws = torch.full((api.qsa_sparse_prefill_workspace_bytes(Nq, max_blocks, w.Hq, Hkv, D, topk),),
                    0x5A, dtype=torch.uint8, device="cuda")
    api.qsa_sparse_prefill(cache, pi["cu_q"].cuda(), b.ctx_lens, int(n_q.max()), pi["q_idx"],
                           pi["k_chunk"], pi["q"], max_blocks, topk, 1.0 / np.sqrt(D), sel, o, lse,
                           ws)
    st, flags = api.qsa_get_device_error()
    assert st == 0, (st, flags)
    torch.cuda.synchronize()
    return sel, o, lse


def check_prefill(b, pi, topk, sel, o, lse):
    w = b.w
    sel, o, lse = sel.cpu().numpy(), o.cpu().numpy(), lse.cpu().numpy()
    q_idx = pi["q_idx"].cpu().numpy()
    qb, qkind = H._bits(pi["q"].cpu())
    q = ref.decode_values(qb, qkind)
    cu = pi["cu_q"].tolist()
    worst = 0.0
    for r in range(w.batch):
        L = int(b.ctx_lens_host[r])
        a = int(b.cu_ctx_host[r])
        k_idx = b.k_idx[a:a + L].cpu().numpy()
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
        nq = cu[r + 1] - cu[r]
        for i in range(nq):
            tok = cu[r] + i
            p = L - nq + i
            want = pre.prefill_token(k_idx, q_idx[tok], q[tok], K, V, p, topk, 1.0 / np.sqrt(w.D))
            assert np.array_equal(sel[tok], want["sel"]), (r, p)
            ma, rl = H.attn_errors(o[tok], want["o"])
            le = H.lse_error(lse[tok], want["lse"])
            assert ma <= H.MAX_ABS and rl <= H.REL_L2 and le <= H.LSE_ABS, (r, p, ma, rl, le)
            worst = max(worst, ma)
    return worst


CASES = [
    # workload, overrides, context lengths, query tokens per request
    ("b32_32k", dict(planted=0), [700, 2503, 3001], [700, 301, 129]),
    ("b32_32k", dict(planted=4), [20000, 6001], [257, 384]),
    ("b32_32k", dict(planted=0, d_idx=64, page_size=16), [5003, 2049], [200, 2049]),
    ("b32_32k", dict(planted=0, d_idx=32, page_size=12), [4099, 3000], [131, 64]),
    ("mixed_fp8", dict(), [9000, 4500], [200, 130]),
    ("b32_32k", dict(planted=0, Hq=32, Hkv=4, topk=256), [7000], [300]),
]


@pytest.mark.parametrize("name,over,lens,n_q", CASES)
def test_sparse_prefill_against_the_oracle(name, over, lens, n_q):
    w = replace(WORKLOADS[name], **over)
    b = make_batch(w, "cuda", ctx_lens=lens, seed=71)
    pi = prefill_inputs(b, n_q, seed=71)
    sel, o, lse = run_prefill(b, pi, b.w.topk)
    check_prefill(b, pi, b.w.topk, sel, o, lse)


def test_prefill_last_token_equals_the_decode_path():
    """The last query token of a chunk is a decode query at the same
    position: same selection row as qsa_index_topk and the same attention
    as the decode step, within the tolerances."""
    w = replace(WORKLOADS["b32_32k"], planted=4)
    b = make_batch(w, "cuda", ctx_lens=[12001, 7000], seed=72)
    pi = prefill_inputs(b, [200, 100], seed=72)
    sel, o, lse = run_prefill(b, pi, w.topk)
    # decode step of the same requests (its last token = the chunk's last)
    b2 = make_batch(w, "cuda", ctx_lens=[12001, 7000], seed=72)
    last = (pi["cu_q"][1:] - 1).long()
    b2.q_idx.copy_(pi["q_idx"][last.cuda()])
    b2.q.copy_(pi["q"][last.cuda()].unsqueeze(1))
    step, _ = H.run_gpu(b2, 1)
    assert torch.equal(step.sel, sel[last.cuda()])
    assert float((step.o[:, 0] - o[last.cuda()]).abs().max()) < 1e-4
