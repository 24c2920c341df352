"""Decode work items longer than a worker warp's metadata piece.

When a batch has more (request, kv head) splits than the decode kernel has
worker warps (148 SMs x 12 on a B200), each split is one work item that the
warp streams in pieces of 128 micro-blocks (bf16) or 256 (fp8), carrying its
online-softmax state across them.  Both batches hold 2048 (request, kv head)
pairs, with contexts from 1200 tokens (some requests keep fewer than 512
blocks, so the last piece is ragged): bf16 over 3 splits of ~171 blocks
(mostly 2 pieces), fp8 over 1 split of up to 512 (2 pieces).  For fp8 the V
scale of every (page, kv head) is multiplied by a power of two that grows
with the page's position, so the power-of-two V reference grows between
pieces and the partial sums are rescaled.  Element-wise parity against the oracle on sampled requests,
properties on every request."""
from dataclasses import replace

import pytest
import torch

import qsa_harness as H
from workloads.qsa_inputs import WORKLOADS, make_batch

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda_and_cleanup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _lens(n: int, seed: int) -> list[int]:
    g = torch.Generator().manual_seed(seed)
    return [int(x) for x in torch.randint(1200, 6000, (n,), generator=g)]


def test_bf16_whole_splits_in_pieces():
    w = replace(WORKLOADS["b128_256k"], planted=0)
    b = make_batch(w, "cuda", ctx_lens=_lens(1024, 11), seed=11)
    step, cache = H.run_gpu(b, 3, keep_scores=False)
    H.check_properties(b, step)
    for r in (0, 511, 1023):
        H.check_request(b, step, cache, r, 3, check_kc=False)
    del step, cache, b


def test_fp8_whole_splits_in_pieces_with_varying_v_scales():
    w = WORKLOADS["mixed_fp8"]
    b = make_batch(w, "cuda", ctx_lens=_lens(512, 12), seed=12)
    # V scale of logical page lp of a request times 2^(min(lp // 4, 12) - 6 + u),
    # u uniform in [-2, 2]: later pieces (later positions) reach larger
    # binades, so every multi-piece item rescales
    g = torch.Generator(device="cpu").manual_seed(12)
    e = torch.zeros(tuple(b.v_scale.shape), dtype=torch.float32)
    P = w.page_size
    for r in range(b.w.batch):
        n_pages = (int(b.ctx_lens_host[r]) + P - 1) // P
        phys = b.block_table_host[r, :n_pages].long()
        lp = torch.arange(n_pages)
        e[phys] = ((lp // 4).clamp(max=12) - 6).to(torch.float32)[:, None]
    e += torch.randint(-2, 3, tuple(e.shape), generator=g).to(torch.float32)
    b.v_scale.mul_(torch.exp2(e).to(b.v_scale.device))
    step, cache = H.run_gpu(b, 1, keep_scores=False)
    H.check_properties(b, step)
    for r in (0, 255, 511):
        H.check_request(b, step, cache, r, 1, check_kc=False)
    del step, cache, b
