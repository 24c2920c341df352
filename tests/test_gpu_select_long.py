"""Selection on long requests with heavy ties.

Requests of 35,000 to 65,536 micro-blocks (the 256k workload's length) with
random keys, with two-valued keys whose scores tie in large groups at the
threshold, with every key equal (every score ties: the exact fallback keeps
the first 512 blocks), and with small topk values against long rows.
Selections and scores must match the oracle bit for bit."""
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


def _check(b, S):
    step, cache = H.run_gpu(b, S)
    for r in range(b.w.batch):
        H.check_request(b, step, cache, r, S)
    H.check_properties(b, step)


def test_random_keys_long_requests():
    # 35,001 .. 65,536 blocks, 8 planted spans each
    w = replace(WORKLOADS["b128_256k"], planted=8)
    _check(make_batch(w, "cuda", ctx_lens=[140001, 262144, 200003], seed=21), 2)


def test_two_valued_keys_many_ties_long_requests():
    # keys +-1, query +-1: even scores in [-512, 512], so many blocks tie at
    # the threshold and are ordered by index
    w = replace(WORKLOADS["b128_256k"], planted=0)
    b = make_batch(w, "cuda", ctx_lens=[140000, 131080], seed=22)
    g = torch.Generator(device="cuda").manual_seed(5)
    b.k_idx.copy_(torch.randint(0, 2, b.k_idx.shape, generator=g, device="cuda", dtype=torch.int8) * 2 - 1)
    b.q_idx.copy_(torch.randint(0, 2, b.q_idx.shape, generator=g, device="cuda", dtype=torch.int8) * 2 - 1)
    _check(b, 2)


def test_all_keys_equal_long_requests():
    # every score ties: the threshold bin overflows shared memory and the
    # exact fallback keeps the first 512 blocks
    w = replace(WORKLOADS["b128_256k"], planted=0)
    b = make_batch(w, "cuda", ctx_lens=[140000, 262144], seed=23)
    b.k_idx.fill_(-7)
    step, cache = H.run_gpu(b, 2)
    assert step.sel[0].cpu().tolist() == list(range(512))
    for r in range(b.w.batch):
        H.check_request(b, step, cache, r, 2)


@pytest.mark.parametrize("topk", [64, 300])
def test_small_topk(topk):
    w = replace(WORKLOADS["b32_32k"], planted=4, topk=topk)
    _check(make_batch(w, "cuda", ctx_lens=[32768, 20001, 77777], seed=24 + topk), 2)


# Requests of more than 262,144 micro-blocks keep their kept blocks in a list
# instead of the shared bitmap, and a topk above 1024 writes that list out
# with a bitonic sort: one request of 1,048,580 tokens (262,145 blocks)
# takes both branches.
@pytest.mark.parametrize("topk", [512, 2048])
def test_requests_beyond_the_bitmap_use_the_kept_list(topk):
    w = replace(WORKLOADS["b128_256k"], planted=8, topk=topk)
    _check(make_batch(w, "cuda", ctx_lens=[1048580, 70001], seed=31), 2)


def test_beyond_the_bitmap_with_every_score_tied():
    # the exact fallback, then the kept list and its bitonic sort
    w = replace(WORKLOADS["b128_256k"], planted=0, topk=2048)
    b = make_batch(w, "cuda", ctx_lens=[1048580, 9000], seed=32)
    b.k_idx.fill_(5)
    step, cache = H.run_gpu(b, 2)
    assert step.sel[0].cpu().tolist() == list(range(2048))
    for r in range(b.w.batch):
        H.check_request(b, step, cache, r, 2)


# More requests than SMs, none longer than 32,768 blocks, take the selection
# in CTAs of 512 threads, two per SM: the group maxima (from 16,384 blocks at
# topk 512), the two passes, and rows shorter than topk, at half the threads.
@pytest.mark.parametrize("topk", [512, 2048])
def test_more_requests_than_sms_take_the_half_size_selection(topk):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    lens = [131072, 100001, 70001, 65537, 33000] + [4099 + 37 * i for i in range(sms)]
    w = replace(WORKLOADS["b128_256k"], planted=8, topk=topk)
    b = make_batch(w, "cuda", ctx_lens=lens, seed=41)
    step, cache = H.run_gpu(b, 2)
    assert H.check_index_every_request(b, step.sel, step.scores) == len(lens)
    for r in (0, 1, 2, 3, 4, len(lens) - 1):
        H.check_request(b, step, cache, r, 2)
    H.check_properties(b, step)
