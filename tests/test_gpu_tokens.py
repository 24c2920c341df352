"""GPU parity of the token-budget selection (qsa_index_topk_tokens) against
the oracle: the kept blocks and the token rows must match bit for bit."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import qsa_harness as H
from oracle import qsa_ref as ref
from sparse_attention_decode_compress_b200 import api
from workloads.qsa_inputs import WORKLOADS, make_batch

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda_and_cleanup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _run_tokens(b, cache, budget):
    B, T = b.w.batch, b.w.T
    max_blocks = H.max_blocks_of(b)
    n_sel = H.step_inputs(b)[3]
    tokens = torch.full((B, budget), 7, dtype=torch.int32, device="cuda")
    sel = torch.full((B, budget // 4), 7, dtype=torch.int32, device="cuda")
    ws = api.new_workspace(api.qsa_index_topk_workspace_bytes(B, max_blocks), "cuda")
    api.qsa_index_topk_tokens(cache, b.q_idx, b.ctx_lens, n_sel, T, max_blocks, budget, tokens,
                              sel, None, ws)
    st, flags = api.qsa_get_device_error()
    assert st == 0, (st, flags)
    return tokens.cpu().numpy(), sel.cpu().numpy()


def _oracle_tokens(b, r, budget):
    L, T = int(b.ctx_lens_host[r]), b.w.T
    a = int(b.cu_ctx_host[r])
    kc = ref.compress_keys(b.k_idx[a:a + L].cpu().numpy())
    scores = ref.block_scores(b.q_idx[r].cpu().numpy(), kc, ref.selection_width(L, T))
    sel = ref.select_blocks(scores, budget // 4)
    return ref.selection_tokens(sel, L, T, budget), sel


CASES = [
    ("b32_32k", [9000, 12345, 4099, 5, 1], 2048),
    ("b32_32k", [3000, 17, 64], 64),
    ("mtp_verify", [16384 + 3, 9001, 12002, 4100], 2048),
    ("mtp_verify", [4102, 7, 5], 16),
]


@pytest.mark.parametrize("name,lens,budget", CASES)
def test_token_budget_matches_oracle(name, lens, budget):
    b = make_batch(WORKLOADS[name], "cuda", ctx_lens=lens, seed=4)
    _, cache = H.run_gpu(b, 2, keep_scores=False)
    tokens, sel = _run_tokens(b, cache, budget)
    for r in range(len(lens)):
        want_tok, want_sel = _oracle_tokens(b, r, budget)
        np.testing.assert_array_equal(sel[r], want_sel)
        np.testing.assert_array_equal(tokens[r], want_tok)


def test_token_budget_ties_take_lowest_blocks():
    """Constant keys: every score ties, the first budget / 4 blocks win
    (exact fallback path of the selection)."""
    w = replace(WORKLOADS["b32_32k"], planted=0)
    b = make_batch(w, "cuda", ctx_lens=[32768, 20000], seed=11)
    b.k_idx.fill_(3)
    _, cache = H.run_gpu(b, 2, keep_scores=False)
    tokens, _ = _run_tokens(b, cache, 2048)
    assert tokens[0].tolist() == list(range(2048))
    for r in range(2):
        np.testing.assert_array_equal(tokens[r], _oracle_tokens(b, r, 2048)[0])


def test_token_budget_host_validation():
    b = make_batch(WORKLOADS["tiny"], "cuda")
    _, cache = H.run_gpu(b, 1, keep_scores=False)
    ws = api.new_workspace(api.qsa_index_topk_workspace_bytes(1, 1024), "cuda")
    for budget in (0, 6, 3):
        tok = torch.empty((1, max(budget, 4)), dtype=torch.int32, device="cuda")
        with pytest.raises((api.QSAError, ValueError)):
            api.qsa_index_topk_tokens(cache, b.q_idx, b.ctx_lens, None, 1, 1024, budget, tok, None,
                                      None, ws)
