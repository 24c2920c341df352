"""Page sizes of any whole number of 4-token micro-blocks (PR #53896 report,
实现拆解: the block size must be divisible by the compress ratio).

Pages of 4, 8, 12, 20 and 36 tokens hold a micro-block count that is not a
multiple of 4, so the indexer's scan reads their rows one by one (a run of 4
rows may cross a page); 48-token pages take the general multiple-of-16 path.
Compressed keys, ring, scores and selections must match the oracle bit for
bit and the attention outputs within tolerance, on every request."""
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


@pytest.mark.parametrize("P,d,T,S", [(4, 128, 1, 2), (8, 128, 1, 3), (12, 64, 1, 2),
                                     (20, 32, 1, 2), (36, 128, 4, 2), (48, 128, 1, 2),
                                     (4, 32, 4, 5), (12, 128, 3, 2)])
def test_page_sizes_divisible_by_the_ratio(P, d, T, S):
    w = replace(WORKLOADS["b32_32k"], page_size=P, d_idx=d, T=T, planted=4)
    b = make_batch(w, "cuda", ctx_lens=[9001, 12345, 4097, 2049], seed=40 + P)
    step, cache = H.run_gpu(b, S)
    for r in range(b.w.batch):
        H.check_request(b, step, cache, r, S)
    H.check_properties(b, step)


def test_page_size_4_one_token_appends():
    """Decode steps one token at a time on 4-token pages: every append
    starts a new page once per micro-block."""
    w = replace(WORKLOADS["b32_32k"], page_size=4, planted=0)
    b = make_batch(w, "cuda", ctx_lens=[3001, 4099], seed=45)
    cache = H.build_cache(b)
    H.prefill(cache, b, 6)
    from sparse_attention_decode_compress_b200 import qsa_compress_append
    for k in range(6, 0, -1):
        pos0 = (b.ctx_lens_host - k).to(torch.int32).cuda()
        rows = torch.tensor([int(b.cu_ctx_host[r + 1]) - k for r in range(2)], device="cuda")
        qsa_compress_append(cache, pos0, torch.tensor([0, 1, 2], dtype=torch.int32, device="cuda"),
                            b.k_idx[rows].contiguous(), 1)
    step, cache = H.run_gpu(b, 2, cache=cache)
    for r in range(2):
        H.check_request(b, step, cache, r, 2)
