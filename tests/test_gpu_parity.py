"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Indexer results (compressed keys, ring, scores,
selected blocks) must match bit for bit; attention outputs within
max-abs 1e-2 / rel-L2 2e-3 and LSE within 1e-4 of the float64 oracle."""
from dataclasses import replace

import numpy as np
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


def _check_all(batch, step, cache, S):
    stats = [H.check_request(batch, step, cache, r, S) for r in range(batch.w.batch)]
    H.check_properties(batch, step)
    return stats


# ------------------------------------------------------------ small sizes --

def test_tiny_workload_exact():
    b = make_batch(WORKLOADS["tiny"], "cuda")
    step, cache = H.run_gpu(b, 1)
    _check_all(b, step, cache, 1)


SMALL = [
    ("b32_32k", [9000, 12345, 4099], 2),
    ("b128_256k", [20000, 8193, 16384], 1),
    ("b128_256k", [20000, 8193, 16384], 4),
    ("mtp_verify", [16384 + 3, 9001, 12002, 4100], 2),
    ("mixed_fp8", [4096, 11111, 30007], 4),
]


@pytest.mark.parametrize("name,lens,S", SMALL)
def test_small_ragged_batches(name, lens, S):
    b = make_batch(WORKLOADS[name], "cuda", ctx_lens=lens, seed=3)
    step, cache = H.run_gpu(b, S)
    _check_all(b, step, cache, S)


@pytest.mark.parametrize("T", [1, 4])
@pytest.mark.parametrize("L", [4, 5, 7, 8, 2047, 2048, 2049, 2052, 2056])
def test_edge_lengths(L, T):
    w = replace(WORKLOADS["b32_32k"], planted=0, T=T)
    b = make_batch(w, "cuda", ctx_lens=[L, 3 * L + 1], seed=L)
    step, cache = H.run_gpu(b, 3)
    _check_all(b, step, cache, 3)


@pytest.mark.parametrize("L", [1, 2, 3])
def test_tiny_contexts(L):
    w = replace(WORKLOADS["b32_32k"], planted=0)
    b = make_batch(w, "cuda", ctx_lens=[L, L + 64], seed=7)
    step, cache = H.run_gpu(b, 2)
    _check_all(b, step, cache, 2)


def test_page_size_16_and_d32_fp32():
    w = replace(WORKLOADS["tiny"], random_table=True)
    b = make_batch(w, "cuda", ctx_lens=[4096, 6001, 333], seed=5)
    step, cache = H.run_gpu(b, 2)
    _check_all(b, step, cache, 2)


def test_all_keys_equal_ties_take_lowest_blocks():
    """Every score ties: the first 512 blocks win (threshold bin overflows
    shared memory -> exact fallback path)."""
    w = replace(WORKLOADS["b32_32k"], planted=0)
    b = make_batch(w, "cuda", ctx_lens=[32768, 20000], seed=11)
    b.k_idx.fill_(3)
    step, cache = H.run_gpu(b, 2)
    assert step.sel[0].cpu().tolist() == list(range(512))
    _check_all(b, step, cache, 2)


def test_two_valued_keys_many_ties():
    w = replace(WORKLOADS["b32_32k"], planted=0)
    b = make_batch(w, "cuda", ctx_lens=[32768, 9999], seed=12)
    g = torch.Generator(device="cuda").manual_seed(1)
    sign = torch.randint(0, 2, b.k_idx.shape, generator=g, device="cuda", dtype=torch.int8)
    b.k_idx.copy_(sign * 2 - 1)
    b.q_idx.fill_(1)
    step, cache = H.run_gpu(b, 2)
    _check_all(b, step, cache, 2)


def test_extreme_scores_order_exactly():
    """Scores at the ends of the int8 range: q = -128 everywhere and 700
    blocks of keys -128 score exactly 2^23 (tied), 300 more score 2^23 - 128,
    the rest mix -128 / 127 / -127.  The selection's ordering keys must span
    the whole score range."""
    w = replace(WORKLOADS["b32_32k"], planted=0)
    b = make_batch(w, "cuda", ctx_lens=[32768, 12000], seed=13)
    g = torch.Generator(device="cuda").manual_seed(2)
    pick = torch.randint(0, 3, b.k_idx.shape, generator=g, device="cuda")
    vals = torch.tensor([-128, 127, -127], dtype=torch.int8, device="cuda")
    b.k_idx.copy_(vals[pick])
    blocks = torch.randperm(32768 // 4, generator=torch.Generator().manual_seed(3))[:1000]
    for j, blk in enumerate(blocks.tolist()):
        rows = b.k_idx[4 * blk:4 * blk + 4]
        rows.fill_(-128)
        if j >= 700:
            rows[0, 0] = -127
    b.q_idx.fill_(-128)
    step, cache = H.run_gpu(b, 2)
    top = sorted(blocks[:700].tolist())[:512]
    assert step.sel[0].cpu().tolist() == top
    _check_all(b, step, cache, 2)


SHAPES = [
    # (workload, overrides, context lengths, splits)
    ("b32_32k", dict(topk=64), [9000, 3001], 2),
    ("b32_32k", dict(topk=2048), [12345, 9001], 2),
    ("b32_32k", dict(topk=4096), [20000, 17000], 3),
    ("b32_32k", dict(D=64), [9000, 5003], 2),
    ("b32_32k", dict(Hq=32, Hkv=4), [9000, 7777], 2),
    ("b32_32k", dict(Hq=8, Hkv=8), [9000, 4097], 2),
    ("b32_32k", dict(Hq=32, Hkv=2), [9000, 6001], 2),
    ("b32_32k", dict(T=2), [9000, 6002], 2),
    ("b32_32k", dict(T=3), [9000, 6003], 2),
    ("b32_32k", dict(page_size=32), [9000, 6007], 2),
    ("b32_32k", dict(d_idx=64), [9000, 6009], 2),
    ("b32_32k", dict(page_size=16, d_idx=32), [9000, 6011], 16),
    ("mixed_fp8", dict(D=64), [9000, 5005], 4),
]


@pytest.mark.parametrize("name,over,lens,S", SHAPES)
def test_other_shapes(name, over, lens, S):
    """Head counts, head and indexer dims, page sizes, query tokens, top-k
    widths and split counts beyond the named workloads."""
    w = replace(WORKLOADS[name], **over)
    b = make_batch(w, "cuda", ctx_lens=lens, seed=17)
    step, cache = H.run_gpu(b, S)
    _check_all(b, step, cache, S)


def test_split_count_invariance():
    w = WORKLOADS["b128_256k"]
    b = make_batch(w, "cuda", ctx_lens=[40000, 30001], seed=21)
    outs = []
    cache = None
    for S in (1, 2, 4, 7):
        step, cache = H.run_gpu(b, S, cache=cache)
        outs.append((step.o.clone(), step.lse.clone(), step.sel.clone()))
        for r in range(2):
            H.check_request(b, step, cache, r, S, check_kc=False)
    for o, lse, sel in outs[1:]:
        assert torch.equal(sel, outs[0][2])
        assert float((o - outs[0][0]).abs().max()) < 1e-4
        assert float((lse - outs[0][1]).abs().max()) < 1e-5


def test_more_splits_than_pages_gives_empty_splits():
    w = replace(WORKLOADS["b32_32k"], planted=0)
    b = make_batch(w, "cuda", ctx_lens=[100, 64], seed=2)   # 2 and 1 pages of 64
    step, cache = H.run_gpu(b, 5)
    _check_all(b, step, cache, 5)
    lse = step.lse_part.cpu()
    assert bool(torch.isneginf(lse[:, 1]).any())


def test_decode_steps_advance_positions():
    """Appending one token at a time keeps the caches equal to the oracle."""
    w = replace(WORKLOADS["b32_32k"], planted=0)
    lens = [3001, 4097]
    b = make_batch(w, "cuda", ctx_lens=lens, seed=9)
    cache = H.build_cache(b)
    H.prefill(cache, b, 6)                 # all but the last 6 positions
    for k in range(6, 0, -1):              # then one position per call
        pos0 = (b.ctx_lens_host - k).to(torch.int32).cuda()
        rows = torch.tensor([int(b.cu_ctx_host[r + 1]) - k for r in range(2)], device="cuda")
        from sparse_attention_decode_compress_b200 import qsa_compress_append
        qsa_compress_append(cache, pos0, torch.tensor([0, 1, 2], dtype=torch.int32, device="cuda"),
                            b.k_idx[rows].contiguous(), 1)
    step, cache = H.run_gpu(b, 2, cache=cache)
    _check_all(b, step, cache, 2)


# ------------------------------------------------------------ error paths --

def test_block_table_out_of_range_reports_bounds():
    from sparse_attention_decode_compress_b200 import qsa_get_device_error
    w = replace(WORKLOADS["b32_32k"], planted=0)
    b = make_batch(w, "cuda", ctx_lens=[4096, 4096], seed=4)
    cache = H.build_cache(b)
    H.prefill(cache, b, 1)
    bad = b.block_table.clone()
    bad[1, 10] = b.num_pages + 7       # not a page: kernels must skip it and report
    cache.block_table = bad
    step, _ = H.run_gpu(b, 2, cache=cache, check_errors=False)
    st, flags = qsa_get_device_error()
    assert st == 3 and (flags & 1)     # QSA_ERR_BOUNDS
    st, flags = qsa_get_device_error()
    assert st == 0 and flags == 0      # cleared
    # request 0 is untouched by the bad entry
    H.check_request(b, step, cache, 0, 2, check_kc=False)


def test_host_validation_rejects_bad_arguments():
    from sparse_attention_decode_compress_b200 import QSAError, qsa_index_topk, qsa_sparse_decode
    w = replace(WORKLOADS["b32_32k"], planted=0)
    b = make_batch(w, "cuda", ctx_lens=[4096], seed=4)
    cache = H.build_cache(b)
    sel = torch.empty((1, 512), dtype=torch.int32, device="cuda")
    ws = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(QSAError, match="INVALID_ARG"):          # workspace too small
        qsa_index_topk(cache, b.q_idx, b.ctx_lens, None, 1024, 512, sel, None, ws)
    with pytest.raises(QSAError, match="INVALID_ARG"):          # topk out of range
        qsa_index_topk(cache, b.q_idx, b.ctx_lens, None, 1024, 5000,
                       torch.empty((1, 5000), dtype=torch.int32, device="cuda"), None, ws)
    o_part = torch.empty((17, 1, 1, 16, 128), device="cuda")
    lse_part = torch.empty((17, 1, 1, 16), device="cuda")
    with pytest.raises(QSAError):                                # 17 splits > 16
        qsa_sparse_decode(cache, b.q, b.ctx_lens, sel, 0.1, 17, o_part, lse_part, ws)


# ------------------------------------------------------------ full sizes --

@pytest.mark.parametrize("name,S", [("b32_32k", 2), ("b128_256k", 2), ("mtp_verify", 2),
                                    ("mixed_fp8", 4)])
def test_full_size(name, S):
    """Full-size workloads in the launch configuration of the benchmark:
    scores and selected blocks bit-exact against the oracle on EVERY
    request; compressed keys, ring and attention element-wise on 16 requests
    spread over the context lengths; properties on every request."""
    b = make_batch(WORKLOADS[name], "cuda")
    step, cache = H.run_gpu(b, S)
    H.check_properties(b, step)
    assert H.check_index_every_request(b, step.sel, step.scores) == b.w.batch
    for r in H.sample_requests(b.ctx_lens_host, 16):
        H.check_request(b, step, cache, r, S)
    del step, cache, b


def test_full_size_256k_split_invariance():
    b = make_batch(WORKLOADS["b128_256k"], "cuda")
    cache = None
    ref_o = None
    for S in (1, 2, 4):
        step, cache = H.run_gpu(b, S, keep_scores=False, cache=cache)
        if ref_o is None:
            ref_o, ref_sel = step.o.clone(), step.sel.clone()
            for r in (0, 77):
                H.check_request(b, step, cache, r, S)
        else:
            assert torch.equal(step.sel, ref_sel)
            assert float((step.o - ref_o).abs().max()) < 1e-4
            H.check_request(b, step, cache, 127, S, check_kc=False)


@pytest.mark.parametrize("name,lens,S", [("b32_32k", [9000, 12345, 4099], 2),
                                         ("mtp_verify", [16384 + 3, 9001], 2),
                                         ("mixed_fp8", [4096, 30007], 4),
                                         ("tiny", None, 1)])
def test_decode_workspace_of_any_contents(name, lens, S):
    """The decode zeroes its workspace header (work counter, split tickets)
    itself: a workspace full of garbage gives the same bits as a zeroed one,
    call after call."""
    from sparse_attention_decode_compress_b200 import api
    b = make_batch(WORKLOADS[name], "cuda", ctx_lens=lens, seed=19)
    step, cache = H.run_gpu(b, S, keep_scores=False)
    for fill in (0xFF, 0x7F, 0x01):
        step.ws_dec.fill_(fill)
        o_part = torch.empty_like(step.o_part)
        lse_part = torch.empty_like(step.lse_part)
        for _ in range(2):
            api.qsa_sparse_decode(cache, b.q, b.ctx_lens, step.sel, step.sm_scale, S, o_part,
                                  lse_part, step.ws_dec)
            st, flags = api.qsa_get_device_error()
            assert st == 0, (fill, st, flags)
            assert torch.equal(o_part, step.o_part) and torch.equal(lse_part, step.lse_part)
