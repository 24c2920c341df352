"""Host-side checks of the seeded input generators (CPU only)."""
import numpy as np
import torch

from oracle import qsa_ref as ref
from workloads.qsa_inputs import WORKLOADS, make_batch, request_pages


def test_tiny_shapes_and_identity_table():
    b = make_batch(WORKLOADS["tiny"], "cpu")
    w = b.w
    assert b.k_cache.shape == (4096 // 16, 16, 1, 64) and b.k_cache.dtype == torch.float32
    assert torch.equal(b.block_table_host[0], torch.arange(256, dtype=torch.int32))
    assert b.k_idx.shape == (4096, 32) and b.k_idx.dtype == torch.int8
    assert int(b.k_idx.min()) >= -127 and int(b.k_idx.max()) <= 127
    assert b.q.shape == (1, 1, 8, 64)


def test_generation_is_seeded():
    a = make_batch(WORKLOADS["tiny"], "cpu")
    b = make_batch(WORKLOADS["tiny"], "cpu")
    assert torch.equal(a.k_cache, b.k_cache) and torch.equal(a.k_idx, b.k_idx)
    c = make_batch(WORKLOADS["tiny"], "cpu", seed=1)
    assert not torch.equal(a.k_idx, c.k_idx)


def test_random_table_is_a_permutation_and_padded():
    b = make_batch(WORKLOADS["mtp_verify"], "cpu", ctx_lens=[4100, 300, 64])
    t = b.block_table_host
    used = t[t >= 0]
    assert sorted(used.tolist()) == list(range(b.num_pages))
    assert (t[1, 5:] == -1).all() and (t[2, 1:] == -1).all()


def test_planted_spans_win_selection():
    b = make_batch(WORKLOADS["b32_32k"], "cpu", ctx_lens=[4096, 5000])
    for r in range(2):
        L = int(b.ctx_lens_host[r])
        a, e = int(b.cu_ctx_host[r]), int(b.cu_ctx_host[r + 1])
        kc = ref.compress_keys(b.k_idx[a:e].numpy())
        s = ref.block_scores(b.q_idx[r].numpy(), kc)
        sel = ref.select_blocks(s, 512)
        assert (b.planted_host[r] >= 0).all()
        assert set(b.planted_host[r].tolist()) <= set(sel.tolist())
        # planted attention keys: scaled logit near 8 for the first query head
        pg = request_pages(b, r)
        K = b.k_cache[pg].reshape(-1, 2, 128)[:L].float()
        t0 = int(b.planted_host[r, 0]) * 4
        logit = (b.q[r, 0, 0].float() @ K[t0, 0]) / np.sqrt(128)
        assert 3.0 < float(logit) < 14.0


def test_fp8_scales_and_codes():
    b = make_batch(WORKLOADS["mixed_fp8"], "cpu", ctx_lens=[4096, 4200])
    assert b.k_cache.dtype == torch.float8_e4m3fn and b.k_scale.shape == (b.num_pages, 4)
    x = b.k_cache.float()
    assert float(x.abs().max()) <= 448.0 and not torch.isnan(x).any()
    amax = x.abs().amax(dim=(1, 3))
    assert torch.allclose(amax, torch.full_like(amax, 448.0))


def test_loguniform_lengths_in_range():
    from workloads.qsa_inputs import draw_ctx_lens
    L = draw_ctx_lens(WORKLOADS["mixed_fp8"], torch.Generator().manual_seed(0))
    assert L.shape == (256,) and int(L.min()) >= 4096 and int(L.max()) <= 1048576


def test_short_requests_get_no_planted_spans():
    b = make_batch(WORKLOADS["b32_32k"], "cpu", ctx_lens=[1, 20, 4096])
    assert (b.planted_host[0] == -1).all() and (b.planted_host[1] == -1).all()
    assert (b.planted_host[2] >= 0).all()
