"""GPU checks of the decode-context-parallel split range: each split computed
alone (qsa_sparse_decode_splits, as one DCP rank would) is bit-identical to
the same split of a full qsa_sparse_decode, and merging the per-rank splits
gives the step's output."""
import numpy as np
import pytest
import torch

import qsa_harness as H
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


# short requests (fewer pages than splits: some of their splits are empty,
# so a rank may see nothing of them) next to long ones
@pytest.mark.parametrize("name,lens,S", [("b32_32k", [9000, 12345, 4099], 2),
                                         ("b32_32k", [100, 9000, 70, 3001], 4),
                                         ("b128_256k", [40000, 30001], 4),
                                         ("mtp_verify", [16384 + 3, 9001], 2),
                                         ("mtp_verify", [131, 5003, 70], 4),
                                         ("mixed_fp8", [4096, 30007], 4)])
def test_split_ranges_match_full_decode(name, lens, S):
    b = make_batch(WORKLOADS[name], "cuda", ctx_lens=lens, seed=8)
    w = b.w
    step, cache = H.run_gpu(b, S, keep_scores=False)
    Hkv, D = b.k_cache.shape[2], b.k_cache.shape[3]
    ranges = [(s, s + 1) for s in range(S)] + ([(1, 3)] if S >= 3 else [])
    o_parts, l_parts = [], []
    for lo, hi in ranges:
        ws = api.new_workspace(api.qsa_sparse_decode_workspace_bytes(w.batch, w.T, w.Hq, Hkv, D,
                                                                     w.topk, S), "cuda")
        o = torch.full((hi - lo,) + tuple(step.o_part.shape[1:]), 7.0, device="cuda")
        l = torch.full((hi - lo,) + tuple(step.lse_part.shape[1:]), 7.0, device="cuda")
        api.qsa_sparse_decode_splits(cache, b.q, b.ctx_lens, step.sel, step.sm_scale, S, lo, hi,
                                     o, l, ws)
        st, flags = api.qsa_get_device_error()
        assert st == 0, (st, flags)
        assert torch.equal(o, step.o_part[lo:hi]), (lo, hi)
        assert torch.equal(l, step.lse_part[lo:hi]), (lo, hi)
        if hi - lo == 1:
            o_parts.append(o)
            l_parts.append(l)
    # what the ranks gather, merged
    o_all, l_all = torch.cat(o_parts), torch.cat(l_parts)
    o_m, l_m = torch.empty_like(step.o), torch.empty_like(step.lse)
    api.qsa_lse_merge(o_all, l_all, o_m, l_m)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(o_m.cpu().numpy(), step.o.cpu().numpy())
    np.testing.assert_array_equal(l_m.cpu().numpy(), step.lse.cpu().numpy())


def test_split_range_rejected_on_host():
    b = make_batch(WORKLOADS["b32_32k"], "cuda", ctx_lens=[5000], seed=2)
    w = b.w
    step, cache = H.run_gpu(b, 2, keep_scores=False)
    ws = api.new_workspace(1 << 24, "cuda")
    for lo, hi in ((1, 1), (-1, 1), (1, 3)):
        n = max(hi - lo, 1)
        o = torch.empty((n,) + tuple(step.o_part.shape[1:]), device="cuda")
        l = torch.empty((n,) + tuple(step.lse_part.shape[1:]), device="cuda")
        with pytest.raises((api.QSAError, ValueError)):
            api.qsa_sparse_decode_splits(cache, b.q, b.ctx_lens, step.sel, step.sm_scale, 2, lo, hi,
                                         o, l, ws)


def _slice_table(b, S: int, s: int) -> torch.Tensor:
    """Block table of a rank that holds only split s's pages: every entry
    outside logical pages [floor(s*NP/S), floor((s+1)*NP/S)) of a request is
    -1 (NP = its page count)."""
    t = b.block_table_host.clone()
    P = b.w.page_size
    for r in range(b.w.batch):
        L = int(b.ctx_lens_host[r])
        NP = (L + P - 1) // P
        lo, hi = s * NP // S, (s + 1) * NP // S
        t[r, :lo] = -1
        t[r, hi:] = -1
    return t.to(b.device)


@pytest.mark.parametrize("name,lens,S", [("b32_32k", [9000, 12345, 4099], 2),
                                         ("b128_256k", [40000, 30001], 4),
                                         ("mtp_verify", [16384 + 3, 9001], 2),
                                         ("mixed_fp8", [4096, 30007], 4)])
def test_rank_slices_against_the_oracle(name, lens, S):
    """Each rank's split, computed with a block table that maps only that
    rank's slice of pages (-1 elsewhere), against the oracle's partials of
    that split; no device error may be raised, and the bits equal those of
    the same split computed with the full table."""
    b = make_batch(WORKLOADS[name], "cuda", ctx_lens=lens, seed=18)
    w = b.w
    step, cache = H.run_gpu(b, S, keep_scores=False)
    Hkv, D = b.k_cache.shape[2], b.k_cache.shape[3]
    want = [H.oracle_request(b, r, S) for r in range(w.batch)]
    o_parts, l_parts = [], []
    for s in range(S):
        rank_cache = api.QSACache(cache.k_cache, cache.v_cache, cache.kc, cache.ring,
                                  _slice_table(b, S, s), cache.k_scale, cache.v_scale)
        ws = api.new_workspace(api.qsa_sparse_decode_workspace_bytes(w.batch, w.T, w.Hq, Hkv, D,
                                                                     w.topk, S), "cuda")
        ws.fill_(0xA5)                     # the call must not rely on a zeroed workspace
        o = torch.full((1,) + tuple(step.o_part.shape[1:]), 7.0, device="cuda")
        l = torch.full((1,) + tuple(step.lse_part.shape[1:]), 7.0, device="cuda")
        api.qsa_sparse_decode_splits(rank_cache, b.q, b.ctx_lens, step.sel, step.sm_scale, S, s,
                                     s + 1, o, l, ws)
        st, flags = api.qsa_get_device_error()
        assert st == 0, (s, st, flags)
        assert torch.equal(o, step.o_part[s:s + 1]) and torch.equal(l, step.lse_part[s:s + 1])
        for r in range(w.batch):
            ma, rl = H.attn_errors(o[0, r].cpu().numpy(), want[r]["o_part"][s])
            le = H.lse_error(l[0, r].cpu().numpy(), want[r]["lse_part"][s])
            assert ma <= H.MAX_ABS and rl <= H.REL_L2 and le <= H.LSE_ABS, (s, r, ma, rl, le)
        o_parts.append(o)
        l_parts.append(l)
    o_m, l_m = torch.empty_like(step.o), torch.empty_like(step.lse)
    api.qsa_lse_merge(torch.cat(o_parts), torch.cat(l_parts), o_m, l_m)
    torch.cuda.synchronize()
    for r in range(w.batch):
        ma, rl = H.attn_errors(o_m[r].cpu().numpy(), want[r]["o"])
        le = H.lse_error(l_m[r].cpu().numpy(), want[r]["lse"])
        assert ma <= H.MAX_ABS and rl <= H.REL_L2 and le <= H.LSE_ABS, (r, ma, rl, le)
