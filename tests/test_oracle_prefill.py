"""Pins of the sparse-prefill oracle (oracle/qsa_ref_prefill.py) against
things other than itself: a hand-worked example, textbook dense causal
attention (scipy) where every block is kept, a brute-force selection written
with explicit loops, the decode oracle at the last token, and causality."""
import json
import math
import os

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

from oracle import qsa_ref as ref
from oracle import qsa_ref_prefill as pre


@pytest.fixture(scope="module")
def hand(golden_dir):
    with open(os.path.join(golden_dir, "prefill_hand.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("topk", [1, 2])
def test_hand_example(hand, topk):
    k = np.array(hand["k_idx"], dtype=np.int8)
    qi = np.array(hand["q_idx"], dtype=np.int8)
    L = k.shape[0]
    K = np.zeros((L, 1, 1))
    V = np.arange(L, dtype=np.float64).reshape(L, 1, 1)
    q = np.ones((L, 1, 1))
    out = pre.prefill_request(k, qi, q, K, V, 0, topk, 1.0)
    for p in range(L):
        assert out["scores"][p].tolist() == hand["scores"][p], p
    assert out["sel"].tolist() == hand[f"topk{topk}_sel"]
    assert np.allclose(out["o"][:, 0, 0], hand[f"topk{topk}_o"], rtol=0, atol=1e-12)
    assert np.allclose(out["lse"][:, 0], np.log(hand[f"topk{topk}_count"]), rtol=0, atol=1e-12)
    if topk == 1:
        for p in range(L):
            toks = ref.token_set(out["sel"][p], p + 1, 1, 0)
            assert toks.tolist() == hand["topk1_tokens"][p]


def _rand(L, d, Hq, Hkv, D, seed):
    rng = np.random.default_rng(seed)
    k = rng.integers(-127, 128, size=(L, d)).astype(np.int8)
    qi = rng.integers(-127, 128, size=(L, d)).astype(np.int8)
    q = rng.standard_normal((L, Hq, D))
    K = rng.standard_normal((L, Hkv, D))
    V = rng.standard_normal((L, Hkv, D))
    return k, qi, q, K, V


def test_every_block_kept_is_dense_causal_attention():
    """With n = floor(p/4) + 1 <= topk every block is kept: token p's output
    is textbook causal softmax attention over tokens 0..p."""
    L, d, Hq, Hkv, D = 61, 8, 4, 2, 16
    k, qi, q, K, V = _rand(L, d, Hq, Hkv, D, 1)
    sm = 1.0 / math.sqrt(D)
    out = pre.prefill_request(k, qi, q, K, V, 0, 16, sm)   # 16 blocks >= ceil(61/4)
    G = Hq // Hkv
    for p in range(L):
        for h in range(Hq):
            x = sm * (K[: p + 1, h // G] @ q[p, h])
            assert np.allclose(out["o"][p, h], softmax(x) @ V[: p + 1, h // G], atol=1e-12)
            assert abs(out["lse"][p, h] - logsumexp(x)) < 1e-12


def test_selection_by_brute_force_loops():
    """Scores and selections against explicit Python loops over tokens and
    dims, with small alphabets so that ties occur."""
    rng = np.random.default_rng(7)
    L, d = 37, 3
    k = rng.integers(-2, 3, size=(L, d)).astype(np.int8)
    qi = rng.integers(-1, 2, size=(L, d)).astype(np.int8)
    for topk in (1, 3, 5):
        for p in range(L):
            nb = p // 4 + 1
            s = []
            for b in range(nb):
                tot = 0
                for t in range(4 * b, min(4 * b + 4, p + 1)):
                    for j in range(d):
                        tot += int(qi[p, j]) * int(k[t, j])
                s.append(tot)
            kc = pre.prefix_block_keys(k, p)
            got = ref.block_scores(qi[p], kc)
            assert got.tolist() == s
            order = sorted(range(nb), key=lambda b: (-s[b], b))[:topk]
            want = sorted(order) + [-1] * (topk - len(order))
            tok = pre.prefill_token(k, qi[p], np.zeros((1, 1)), np.zeros((L, 1, 1)),
                                    np.zeros((L, 1, 1)), p, topk, 1.0)
            assert tok["sel"].tolist() == want, (topk, p)


def test_last_token_equals_the_decode_oracle():
    L, d, Hq, Hkv, D = 2200, 16, 4, 1, 8
    k, qi, q, K, V = _rand(L, d, Hq, Hkv, D, 3)
    sm = 1.0 / math.sqrt(D)
    tok = pre.prefill_token(k, qi[L - 1], q[L - 1], K, V, L - 1, 64, sm)
    dec = ref.decode_request(k, qi[L - 1], q[L - 1:L], K, V, 1, 16, 1, 64, sm)
    assert np.array_equal(tok["sel"], dec["sel"])
    assert np.allclose(tok["o"], dec["o"][0], atol=1e-12)
    assert np.allclose(tok["lse"], dec["lse"][0], atol=1e-12)


def test_tokens_do_not_see_later_tokens():
    L, d, Hq, Hkv, D = 300, 8, 2, 1, 8
    k, qi, q, K, V = _rand(L, d, Hq, Hkv, D, 4)
    p = 201                                         # mid-block: its block sums 2 tokens
    a = pre.prefill_token(k, qi[p], q[p], K, V, p, 8, 0.3)
    k2, K2, V2 = k.copy(), K.copy(), V.copy()
    k2[p + 1:] = 127
    K2[p + 1:] = 9.0
    V2[p + 1:] = -9.0
    b = pre.prefill_token(k2, qi[p], q[p], K2, V2, p, 8, 0.3)
    assert np.array_equal(a["scores"], b["scores"]) and np.array_equal(a["sel"], b["sel"])
    assert np.array_equal(a["o"], b["o"]) and np.array_equal(a["lse"], b["lse"])
    # ... while the full cache's block sum (all 4 tokens) would differ
    assert not np.array_equal(ref.compress_keys(k2)[p // 4], pre.prefix_block_keys(k2, p)[p // 4])
