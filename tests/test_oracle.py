"""Pins for the CPU oracle: every function is checked against something other
than itself (a hand-worked example, a closed form, brute force, or a library
routine), chosen so that a dropped term, a wrong sign or index, or a swapped
operand fails at least one test."""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp, softmax

from oracle import qsa_ref as ref


# --------------------------------------------------------------------------
# Hand-worked example (tests/golden/hand_example.json)
# --------------------------------------------------------------------------

@pytest.fixture(scope="module")
def hand(golden_dir):
    with open(os.path.join(golden_dir, "hand_example.json")) as f:
        return json.load(f)


def _f(x):
    return -math.inf if x == "-inf" else float(x)


def test_hand_compress_scores_select(hand):
    k = np.array(hand["k_idx"], dtype=np.int8)
    kc = ref.compress_keys(k)
    assert kc.tolist() == hand["kc"]
    s = ref.block_scores(np.array(hand["q_idx"], dtype=np.int8), kc)
    assert s.tolist() == hand["scores"]
    for kk in (1, 2, 4):
        assert ref.select_blocks(s, kk).tolist()[:kk] == hand[f"sel_topk{kk}"][:kk]
        assert ref.select_blocks(s, 4).tolist() == hand["sel_topk4"]
    assert ref.select_blocks(s, 4).tolist() == hand["sel_topk4"]
    assert ref.select_blocks(s, 2).tolist() + [-1, -1] == hand["sel_topk2"]
    s0 = ref.block_scores(np.array(hand["tie_q_idx"], dtype=np.int8), kc)
    assert ref.select_blocks(s0, 2).tolist() + [-1, -1] == hand["tie_sel_topk2"]


def test_hand_attention_and_splits(hand):
    L = len(hand["attn_K"])
    K = np.array(hand["attn_K"], dtype=np.float64).reshape(L, 1, 1)
    V = np.array(hand["attn_V"], dtype=np.float64).reshape(L, 1, 1)
    q = np.array([[hand["attn_q"]]])
    sel = np.array(hand["attn_sel"] + [-1, -1], dtype=np.int32)
    toks = ref.token_set(sel, L, 1, 0)
    assert toks.tolist() == [4, 5, 6, 7, 8]
    o, lse = ref.attention(q, K, V, toks, hand["attn_scale"])
    assert abs(o[0, 0] - hand["attn_o"]) < 1e-12
    assert abs(lse[0] - hand["attn_lse"]) < 1e-12
    P = hand["split_page_size"]
    for S in (2, 3):
        op, lp = ref.split_attention(q, K, V, toks, hand["attn_scale"], L, P, S)
        exp_o = hand[f"split_S{S}_o"]
        exp_l = [_f(x) for x in hand[f"split_S{S}_lse"]]
        for s in range(S):
            assert abs(op[s, 0, 0] - exp_o[s]) < 1e-12
            if math.isinf(exp_l[s]):
                assert lp[s, 0] == -math.inf
            else:
                assert abs(lp[s, 0] - exp_l[s]) < 1e-12
        om, lm = ref.lse_merge(op, lp)
        assert abs(om[0, 0] - hand["attn_o"]) < 1e-12
        assert abs(lm[0] - hand["attn_lse"]) < 1e-12


def test_hand_mtp(hand):
    k = np.array(hand["k_idx"], dtype=np.int8)
    L, T = k.shape[0], hand["mtp_T"]
    kc = ref.compress_keys(k)
    n_sel = ref.selection_width(L, T)
    assert n_sel == 2
    s = ref.block_scores(np.array(hand["q_idx"], dtype=np.int8), kc, n_sel)
    sel = ref.select_blocks(s, 1)
    assert sel.tolist() == hand["mtp_sel_topk1"]
    assert ref.token_set(sel, L, T, 0).tolist() == hand["mtp_tokens_t0"]
    assert ref.token_set(sel, L, T, 1).tolist() == hand["mtp_tokens_t1"]


def test_hand_token_budget(hand):
    k = np.array(hand["k_idx"], dtype=np.int8)
    L = k.shape[0]
    s = ref.block_scores(np.array(hand["q_idx"], dtype=np.int8), ref.compress_keys(k))
    assert ref.selection_tokens(ref.select_blocks(s, 2), L, 1, 8).tolist() == hand["budget8_tokens_T1"]
    assert ref.selection_tokens(ref.select_blocks(s, 4), L, 1, 16).tolist() == hand["budget16_tokens_T1"]
    T = hand["mtp_T"]
    s_mtp = ref.block_scores(np.array(hand["q_idx"], dtype=np.int8), ref.compress_keys(k),
                             ref.selection_width(L, T))
    assert ref.selection_tokens(ref.select_blocks(s_mtp, 1), L, T, 4).tolist() == hand["budget4_tokens_mtp"]


def test_token_budget_properties_brute_force():
    """Every listed token lies in a selected block and at or before p0; the
    row is ascending with its -1 at the end; nothing visible is left out;
    the listed tokens are query token 0's attended set."""
    rng = np.random.default_rng(5)
    for _ in range(300):
        L = int(rng.integers(1, 60))
        T = int(rng.integers(1, 5))
        n = (L + 3) // 4
        topk = int(rng.integers(1, 12))
        sel = ref.select_blocks(rng.integers(-5, 5, n), topk)
        budget = 4 * topk
        row = ref.selection_tokens(sel, L, T, budget)
        p0 = L - T
        kept = [int(b) for b in sel if b >= 0]
        listed = [int(t) for t in row if t >= 0]
        expect = [4 * b + j for b in kept for j in range(4) if 4 * b + j <= p0]
        assert listed == sorted(expect)
        assert all(t == -1 for t in row[len(listed):])
        assert all(t // 4 in kept and t <= p0 for t in listed)
        assert listed == ref.token_set(sel, L, T, 0).tolist()


# --------------------------------------------------------------------------
# Value decoding vs the library conversions
# --------------------------------------------------------------------------

def test_bf16_decode_all_codes():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    mine = ref.bf16_bits_to_f64(bits)
    lib = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().double().numpy()
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], lib[~nan])


def test_e4m3_decode_all_codes():
    bits = np.arange(256, dtype=np.uint8)
    mine = ref.e4m3_bits_to_f64(bits)
    lib = torch.from_numpy(bits).view(torch.float8_e4m3fn).float().double().numpy()
    nan = np.isnan(lib)
    assert nan.sum() == 2                       # S.1111.111 only
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], lib[~nan])
    assert np.nanmax(mine) == 448.0 and np.nanmin(mine[mine > 0]) == 2.0 ** -9


# --------------------------------------------------------------------------
# Compression
# --------------------------------------------------------------------------

@pytest.mark.parametrize("L", [1, 3, 4, 5, 8, 9, 63, 64, 65])
def test_compress_brute_force_and_invariants(L):
    rng = np.random.default_rng(L)
    d = 6
    k = rng.integers(-128, 128, size=(L, d)).astype(np.int8)
    kc = ref.compress_keys(k)
    # brute force scatter: token t contributes to block t // 4
    bf = [[0] * d for _ in range((L + 3) // 4)]
    for t in range(L):
        for j in range(d):
            bf[t // 4][j] += int(k[t, j])
    assert kc.tolist() == bf
    # conservation: every token counted exactly once
    assert np.array_equal(kc.sum(axis=0), k.astype(np.int64).sum(axis=0))
    assert kc.shape[0] == math.ceil(L / 4)


def test_compress_one_hot_locality():
    L, d = 23, 3
    for t in range(L):
        k = np.zeros((L, d), dtype=np.int8)
        k[t, 1] = 7
        kc = ref.compress_keys(k)
        nz = np.argwhere(kc != 0)
        assert nz.tolist() == [[t // 4, 1]]
        assert kc[t // 4, 1] == 7


def test_compress_extremes_fit_ten_bits():
    # the range the packed 10-bit cache layout must hold: [-512, 508]
    k = np.full((8, 4), -128, dtype=np.int8)
    assert ref.compress_keys(k).min() == -512
    k = np.full((8, 4), 127, dtype=np.int8)
    assert ref.compress_keys(k).max() == 508


# --------------------------------------------------------------------------
# Scores
# --------------------------------------------------------------------------

def test_scores_vs_float_matmul_and_loops():
    rng = np.random.default_rng(1)
    kc = rng.integers(-512, 509, size=(300, 128))
    q = rng.integers(-128, 128, size=128).astype(np.int8)
    s = ref.block_scores(q, kc)
    f = np.dot(kc.astype(np.float64), q.astype(np.float64))  # exact: all sums < 2^53
    assert np.array_equal(s, f.astype(np.int64))
    for b in (0, 17, 299):
        assert s[b] == sum(int(kc[b, j]) * int(q[j]) for j in range(128))
    assert ref.block_scores(q, kc, 10).shape == (10,)


def test_scores_one_hot_query_reads_column():
    kc = np.arange(40).reshape(10, 4) - 20
    q = np.array([0, 0, 1, 0], dtype=np.int8)
    assert np.array_equal(ref.block_scores(q, kc), kc[:, 2])
    q = np.array([0, -1, 0, 0], dtype=np.int8)
    assert np.array_equal(ref.block_scores(q, kc), -kc[:, 1])


# --------------------------------------------------------------------------
# Selection
# --------------------------------------------------------------------------

def _brute_select(scores, k):
    n = len(scores)
    order = sorted(range(n), key=lambda b: (-int(scores[b]), b))
    keep = sorted(order[:min(k, n)])
    return keep + [-1] * (k - len(keep))


@pytest.mark.parametrize("seed", range(12))
def test_select_vs_full_sort(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 65))
    k = int(rng.integers(1, 70))
    alphabet = [2, 3, 1000][seed % 3]            # small alphabets: many ties
    s = rng.integers(-alphabet // 2, alphabet // 2 + 1, size=n)
    assert ref.select_blocks(s, k).tolist() == _brute_select(s, k)


def test_select_constant_scores_take_lowest_indices():
    s = np.full(5000, 42)
    assert ref.select_blocks(s, 512).tolist() == list(range(512))


def test_select_fewer_blocks_than_budget_pads():
    s = np.array([5, -1, 3])
    assert ref.select_blocks(s, 6).tolist() == [0, 1, 2, -1, -1, -1]
    assert ref.select_blocks(np.array([], dtype=np.int64), 3).tolist() == [-1, -1, -1]


def test_select_planted_maxima():
    rng = np.random.default_rng(5)
    s = rng.integers(-1000, 1000, size=4096)
    planted = [7, 100, 2047, 4095]
    s[planted] = 10 ** 6
    sel = ref.select_blocks(s, 8)
    assert set(planted) <= set(sel.tolist())


# --------------------------------------------------------------------------
# Token sets
# --------------------------------------------------------------------------

def test_token_set_decode_and_tail_block():
    sel = np.array([0, 2, -1], dtype=np.int32)
    assert ref.token_set(sel, 10, 1, 0).tolist() == [0, 1, 2, 3, 8, 9]
    sel = np.array([1, -1], dtype=np.int32)
    assert ref.token_set(sel, 6, 1, 0).tolist() == [4, 5]


def test_token_set_mtp_union_no_double_count():
    # L = 12, T = 4: p0 = 8; block 2 (tokens 8..11) holds p0 and all spec tokens
    sel = np.array([2, 0], dtype=np.int32)
    assert ref.token_set(sel, 12, 4, 0).tolist() == [0, 1, 2, 3, 8]
    assert ref.token_set(sel, 12, 4, 3).tolist() == [0, 1, 2, 3, 8, 9, 10, 11]
    # block 2 not selected: the tail (8, p_t] is still attended, p0 itself is not
    sel = np.array([0], dtype=np.int32)
    assert ref.token_set(sel, 12, 4, 0).tolist() == [0, 1, 2, 3]
    assert ref.token_set(sel, 12, 4, 2).tolist() == [0, 1, 2, 3, 9, 10]


# --------------------------------------------------------------------------
# Attention, splits, merge
# --------------------------------------------------------------------------

def _dense(q, K, V, scale, upto=None):
    """Textbook softmax(q K^T * scale) V via scipy, GQA by head grouping."""
    Hq, D = q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    n = K.shape[0] if upto is None else upto
    o = np.zeros((Hq, D))
    lse = np.zeros(Hq)
    for h in range(Hq):
        x = scale * np.einsum("d,td->t", q[h], K[:n, h // G])
        o[h] = softmax(x) @ V[:n, h // G]
        lse[h] = logsumexp(x)
    return o, lse


def test_attention_closed_forms():
    rng = np.random.default_rng(3)
    L, Hq, Hkv, D = 9, 4, 2, 8
    q = rng.standard_normal((Hq, D))
    K = rng.standard_normal((L, Hkv, D))
    V = np.broadcast_to(rng.standard_normal((1, Hkv, D)), (L, Hkv, D)).copy()
    toks = np.arange(L)
    o, _ = ref.attention(q, K, V, toks, 0.3)
    for h in range(Hq):                              # constant V -> o = v
        assert np.allclose(o[h], V[0, h // 2], atol=1e-13)
    one = np.array([5])
    o, lse = ref.attention(q, K, rng.standard_normal((L, Hkv, D)), one, 0.3)
    assert np.allclose(lse, 0.3 * np.einsum("hd,hd->h", q, K[5, [0, 0, 1, 1]]), atol=1e-13)
    Kz = np.zeros((L, Hkv, D))                      # equal logits -> mean, lse = log n
    V2 = rng.standard_normal((L, Hkv, D))
    o, lse = ref.attention(q, Kz, V2, toks, 0.3)
    assert np.allclose(o[0], V2.mean(axis=0)[0], atol=1e-13)
    assert np.allclose(lse, math.log(L), atol=1e-13)
    o, lse = ref.attention(q, K, V2, np.array([], dtype=np.int64), 0.3)
    assert np.all(o == 0) and np.all(lse == -np.inf)


def test_attention_vs_textbook_dense():
    rng = np.random.default_rng(4)
    L, Hq, Hkv, D = 37, 8, 2, 16
    q = rng.standard_normal((Hq, D))
    K = rng.standard_normal((L, Hkv, D)) * 2
    V = rng.standard_normal((L, Hkv, D))
    o, lse = ref.attention(q, K, V, np.arange(L), 1 / math.sqrt(D))
    o2, lse2 = _dense(q, K, V, 1 / math.sqrt(D))
    assert np.allclose(o, o2, atol=1e-12) and np.allclose(lse, lse2, atol=1e-12)


def test_split_bounds_cover_pages():
    for L in (1, 5, 64, 65, 1000):
        for P in (4, 16, 64):
            for S in (1, 2, 3, 4, 7):
                b = ref.split_bounds(L, P, S)
                assert b[0] == 0 and b[-1] == L and np.all(np.diff(b) >= 0)
                assert np.all((b[1:-1] % P == 0) | (b[1:-1] == L))


@pytest.mark.parametrize("S", [1, 2, 4])
def test_merge_of_splits_equals_unsplit(S):
    rng = np.random.default_rng(S)
    L, Hq, Hkv, D, P = 300, 8, 2, 16, 16
    q = rng.standard_normal((Hq, D))
    K = rng.standard_normal((L, Hkv, D))
    V = rng.standard_normal((L, Hkv, D))
    toks = np.sort(rng.choice(L, 120, replace=False))
    o, lse = ref.attention(q, K, V, toks, 0.25)
    op, lp = ref.split_attention(q, K, V, toks, 0.25, L, P, S)
    om, lm = ref.lse_merge(op, lp)
    assert np.allclose(om, o, atol=1e-12) and np.allclose(lm, lse, atol=1e-12)
    # merge formula vs scipy logsumexp on the partials
    assert np.allclose(logsumexp(lp, axis=0), lm, atol=1e-12)


def test_merge_empty_split_is_identity_and_all_empty():
    rng = np.random.default_rng(9)
    o = rng.standard_normal((1, 3, 4))
    lse = rng.standard_normal((1, 3))
    op = np.concatenate([o, np.zeros_like(o)])
    lp = np.concatenate([lse, np.full_like(lse, -np.inf)])
    om, lm = ref.lse_merge(op, lp)
    assert np.allclose(om, o[0]) and np.allclose(lm, lse[0])
    om, lm = ref.lse_merge(np.zeros((3, 2, 4)), np.full((3, 2), -np.inf))
    assert np.all(om == 0) and np.all(lm == -np.inf)


# --------------------------------------------------------------------------
# Whole path: sparse == dense when everything is selected
# --------------------------------------------------------------------------

def _rand_request(rng, L, d, Hq, Hkv, D, T=1):
    k_idx = rng.integers(-127, 128, size=(L, d)).astype(np.int8)
    q_idx = rng.integers(-127, 128, size=d).astype(np.int8)
    q = rng.standard_normal((T, Hq, D))
    K = rng.standard_normal((L, Hkv, D))
    V = rng.standard_normal((L, Hkv, D))
    return k_idx, q_idx, q, K, V


@pytest.mark.parametrize("L", [1, 3, 4, 5, 2047, 2048])
def test_all_selected_equals_dense(L):
    rng = np.random.default_rng(L)
    Hq, Hkv, D = 4, 2, 8
    k_idx, q_idx, q, K, V = _rand_request(rng, L, 8, Hq, Hkv, D)
    out = ref.decode_request(k_idx, q_idx, q, K, V, T=1, page_size=16, num_splits=2)
    n = math.ceil(L / 4)
    assert out["sel"][:n].tolist() == list(range(n))
    o2, lse2 = _dense(q[0], K, V, 1 / math.sqrt(D))
    assert np.allclose(out["o"][0], o2, atol=1e-12)
    assert np.allclose(out["lse"][0], lse2, atol=1e-12)
    assert np.allclose(out["o_merged"][0], o2, atol=1e-12)


def test_more_than_budget_is_sparse():
    rng = np.random.default_rng(11)
    L = 2049                                    # 513 blocks > 512
    k_idx, q_idx, q, K, V = _rand_request(rng, L, 8, 2, 1, 8)
    out = ref.decode_request(k_idx, q_idx, q, K, V, T=1, page_size=16, num_splits=1)
    assert (out["sel"] >= 0).sum() == 512
    dropped = sorted(set(range(513)) - set(out["sel"].tolist()))
    assert len(dropped) == 1
    s = out["scores"]
    assert s[dropped[0]] == s.min()


def test_mtp_all_selected_equals_dense_causal():
    rng = np.random.default_rng(12)
    L, T, Hq, Hkv, D = 203, 4, 4, 2, 8
    k_idx, q_idx, q, K, V = _rand_request(rng, L, 8, Hq, Hkv, D, T)
    out = ref.decode_request(k_idx, q_idx, q, K, V, T=T, page_size=16, num_splits=4)
    for t in range(T):
        o2, lse2 = _dense(q[t], K, V, 1 / math.sqrt(D), upto=L - T + t + 1)
        assert np.allclose(out["o"][t], o2, atol=1e-12)
        assert np.allclose(out["o_merged"][t], o2, atol=1e-12)
        assert np.allclose(out["lse_merged"][t], lse2, atol=1e-12)


def test_mtp_token0_equals_plain_decode_when_block_aligned():
    rng = np.random.default_rng(13)
    L, T = 4 * 700 + 3, 4                   # p0 + 1 = L - 3 = 2800, a multiple of 4
    Hq, Hkv, D = 4, 1, 8
    k_idx, q_idx, q, K, V = _rand_request(rng, L, 8, Hq, Hkv, D, T)
    mtp = ref.decode_request(k_idx, q_idx, q, K, V, T=T, page_size=16, num_splits=1)
    Lp = L - T + 1
    plain = ref.decode_request(k_idx[:Lp], q_idx, q[:1], K[:Lp], V[:Lp], T=1, page_size=16,
                               num_splits=1)
    assert np.array_equal(mtp["sel"], plain["sel"])
    assert np.allclose(mtp["o"][0], plain["o"][0], atol=1e-13)
    assert np.allclose(mtp["lse"][0], plain["lse"][0], atol=1e-13)


def test_depage_roundtrip():
    rng = np.random.default_rng(14)
    P, L = 8, 29
    npg = math.ceil(L / P)
    logical = rng.standard_normal((npg * P, 2, 3))
    perm = rng.permutation(10)[:npg]
    cache = np.zeros((10, P, 2, 3))
    for i, p in enumerate(perm):
        cache[p] = logical[i * P:(i + 1) * P]
    assert np.array_equal(ref.depage(cache, perm, L, P), logical[:L])
    kc_logical = rng.integers(-5, 5, size=(npg * P // 4, 3))
    kc_cache = np.zeros((10, P // 4, 3), dtype=np.int64)
    for i, p in enumerate(perm):
        kc_cache[p] = kc_logical[i * 2:(i + 1) * 2]
    assert np.array_equal(ref.depage_kc(kc_cache, perm, L, P), kc_logical[:math.ceil(L / 4)])


def test_stored_rows_decode_matches_eager():
    rng = np.random.default_rng(21)
    L, Hkv, D = 11, 2, 4
    bits = rng.integers(0, 256, size=(L, Hkv, D)).astype(np.uint8)
    bits[bits == 0x7F] = 0x11
    bits[bits == 0xFF] = 0x91
    scale = rng.random((L, Hkv)) + 0.5
    view = ref.StoredRows(bits, "e4m3", scale)
    eager = ref.e4m3_bits_to_f64(bits) * scale[..., None]
    toks = np.array([0, 3, 10])
    assert np.array_equal(view[toks, 1, :], eager[toks, 1, :])
    b16 = rng.integers(0, 1 << 16, size=(L, Hkv, D)).astype(np.uint16)
    b16 = (b16 & 0x3FFF).astype(np.uint16)          # finite values only
    v16 = ref.StoredRows(b16, "bf16")
    assert np.array_equal(v16[toks, 0, :], ref.bf16_bits_to_f64(b16)[toks, 0, :])
    assert v16.shape == (L, Hkv, D)
