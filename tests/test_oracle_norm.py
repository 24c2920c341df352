"""Pins of the normalised-pooling indexer oracle (oracle/qsa_ref_norm.py)
against closed forms, the pinned integer oracle, a library RMS norm and brute
force."""
import numpy as np
import pytest
import torch

from oracle import qsa_ref as ref
from oracle import qsa_ref_norm as nrm


def test_pool_mean_closed_forms_and_tail():
    rng = np.random.default_rng(0)
    k = rng.normal(size=(10, 8))
    p = nrm.pool_mean(k)
    assert p.shape == (3, 8)
    assert np.allclose(p[0], (k[0] + k[1] + k[2] + k[3]) / 4, rtol=0, atol=1e-15)
    assert np.allclose(p[2], (k[8] + k[9]) / 2, rtol=0, atol=1e-15)   # tail of 2 tokens
    same = np.tile(k[:1], (4, 1))
    assert np.array_equal(nrm.pool_mean(same)[0], k[0])


def test_pool_mean_is_the_integer_sum_over_four_for_full_blocks():
    rng = np.random.default_rng(1)
    k = rng.integers(-128, 128, size=(64, 32)).astype(np.int8)
    assert np.array_equal(nrm.pool_mean(k) * 4, ref.compress_keys(k).astype(np.float64))


def test_rms_normalise_closed_forms():
    for c in (3.0, -0.5, 1e-4):
        y = nrm.rms_normalise(np.full(16, c))
        assert np.allclose(y, c / np.sqrt(c * c + nrm.RMS_EPS), rtol=1e-15, atol=0)
    rng = np.random.default_rng(2)
    x = rng.normal(size=(5, 64))
    y = nrm.rms_normalise(x, eps=0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-14)
    assert np.allclose(nrm.rms_normalise(7.5 * x, eps=0.0), y, rtol=1e-14)   # scale invariant
    w = rng.normal(size=64) * 0.1
    assert np.allclose(nrm.rms_normalise(x, weight=w), nrm.rms_normalise(x) * (1 + w), rtol=1e-15)


def test_rms_normalise_matches_torch_rms_norm():
    rng = np.random.default_rng(3)
    x = rng.normal(size=(7, 128))
    w = rng.normal(size=128) * 0.2
    lib = torch.nn.functional.rms_norm(torch.from_numpy(x), (128,), torch.from_numpy(1 + w),
                                       eps=nrm.RMS_EPS).numpy()
    assert np.allclose(nrm.rms_normalise(x, weight=w), lib, rtol=1e-13, atol=1e-15)


def test_compressed_key_ignores_the_scale_of_a_block():
    rng = np.random.default_rng(4)
    k = rng.normal(size=(8, 32))
    k2 = k.copy()
    k2[4:8] *= 9.0                     # block 1 scaled up
    a, b = nrm.compress_keys_norm(k, eps=0.0), nrm.compress_keys_norm(k2, eps=0.0)
    assert np.allclose(a, b, rtol=1e-14)


def test_scores_and_selection_brute_force():
    rng = np.random.default_rng(5)
    kc = rng.normal(size=(200, 16))
    q = rng.normal(size=16)
    s = nrm.block_scores_f(q, kc)
    for b in (0, 99, 199):
        assert s[b] == pytest.approx(sum(q[j] * kc[b, j] for j in range(16)), rel=1e-13)
    # integer-valued float scores with ties: same rows as the integer oracle
    si = rng.integers(-5, 6, size=300)
    got = nrm.select_blocks_f(si.astype(np.float64), 64)
    assert np.array_equal(got, ref.select_blocks(si, 64))
    brute = sorted(sorted(range(300), key=lambda i: (-si[i], i))[:64])
    assert got.tolist() == brute
    assert nrm.select_blocks_f(np.ones(5), 8).tolist() == [0, 1, 2, 3, 4, -1, -1, -1]


def test_selection_within_tolerance():
    s = np.array([5.0, 4.0, 3.0, 2.9999999, 1.0, 0.0])
    exact = nrm.select_blocks_f(s, 3)
    assert exact.tolist() == [0, 1, 2]
    assert nrm.selection_within_tolerance(exact, s, 3, atol=1e-6)
    assert nrm.selection_within_tolerance(np.array([0, 1, 3]), s, 3, atol=1e-6)   # near tie
    assert not nrm.selection_within_tolerance(np.array([0, 1, 4]), s, 3, atol=1e-6)  # far
    assert not nrm.selection_within_tolerance(np.array([1, 0, 2]), s, 3, atol=1e-6)  # order
    assert not nrm.selection_within_tolerance(np.array([0, 1, -1]), s, 3, atol=1e-6)  # count
    assert nrm.selection_within_tolerance(np.array([0, 1, -1, -1]), s[:2], 4, atol=0.0)
