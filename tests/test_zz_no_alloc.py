"""The allocation-free indexer entry point (qsa_index_topk_noalloc).

Some callers cannot give the library device memory of their own: a plugin
inside a framework that owns every allocation, or a latency-critical path
where cudaMalloc would synchronise the device.  This entry point keeps its
scores in a fixed array inside libqsa.so instead of a caller workspace.  Its
selections must equal the oracle's and those of qsa_index_topk, on calls in
a row that reuse the shared array, including a call that follows a larger
call with different keys (so it must overwrite stale scores).  This file is
collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import qsa_harness as H
from oracle import qsa_ref as ref
from sparse_attention_decode_compress_b200 import _lib
from workloads.qsa_inputs import WORKLOADS, make_batch

pytestmark = pytest.mark.gpu


def _call_noalloc(cache, q_idx, ctx_lens, n_sel, max_blocks, topk, sel):
    lib = _lib.load()
    s = cache.struct()
    stream = torch.cuda.current_stream().cuda_stream
    return lib.qsa_index_topk_noalloc(ctypes.byref(s), q_idx.shape[0], q_idx.data_ptr(),
                                      ctx_lens.data_ptr(),
                                      None if n_sel is None else n_sel.data_ptr(),
                                      max_blocks, topk, sel.data_ptr(), stream)


def _noalloc(b, cache, n_sel):
    sel = torch.full((b.w.batch, b.w.topk), -7, dtype=torch.int32, device="cuda")
    st = _call_noalloc(cache, b.q_idx, b.ctx_lens, n_sel, H.max_blocks_of(b), b.w.topk, sel)
    assert st == 0, _lib.load().qsa_status_string(st)
    torch.cuda.synchronize()
    return sel


def _oracle_sel(b, r):
    a, e = int(b.cu_ctx_host[r]), int(b.cu_ctx_host[r + 1])
    kc = ref.compress_keys(b.k_idx[a:e].cpu().numpy())
    L = e - a
    scores = ref.block_scores(b.q_idx[r].cpu().numpy(), kc, ref.selection_width(L, b.w.T))
    return ref.select_blocks(scores, b.w.topk)


@pytest.mark.parametrize("name,lens", [("b32_32k", [32768, 9000, 4099, 1]),
                                       ("mtp_verify", [16384 + 3, 9001, 4100])])
def test_noalloc_matches_oracle_and_workspace_entry_point(name, lens):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    # a larger call first, with other keys: it fills more of the shared
    # array than the checked calls use, with scores that must not survive
    big = make_batch(WORKLOADS["b32_32k"], "cuda", ctx_lens=[65536, 65536, 65536, 65536, 65536],
                     seed=99)
    big_cache = H.build_cache(big)
    H.prefill(big_cache, big, 0)
    _noalloc(big, big_cache, None)

    b = make_batch(WORKLOADS[name], "cuda", ctx_lens=lens, seed=17)
    step, cache = H.run_gpu(b, 2)           # the workspace entry point (qsa_index_topk)
    want = step.sel.clone()
    _, _, _, n_sel = H.step_inputs(b)
    for _ in range(2):                      # two calls in a row share the static array
        got = _noalloc(b, cache, n_sel)
        assert torch.equal(got, want)       # indices: bit-exact against qsa_index_topk
        got_h = got.cpu().numpy()
        for r in range(b.w.batch):          # ... and against the oracle
            assert np.array_equal(got_h[r], _oracle_sel(b, r)), r


def test_noalloc_rejects_too_many_scores():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    b = make_batch(WORKLOADS["b32_32k"], "cuda", ctx_lens=[4096], seed=3)
    cache = H.build_cache(b)
    sel = torch.empty((1, 512), dtype=torch.int32, device="cuda")
    st = _call_noalloc(cache, b.q_idx, b.ctx_lens, None, 8 * 1024 * 1024 + 1, 512, sel)
    assert st == 2                          # QSA_ERR_UNSUPPORTED, nothing launched
