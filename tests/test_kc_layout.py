"""The packed compressed-key page layout of include/qsa.h
(qsa_kc_page_bytes): page sizes from the library, and the test harness's
reader of the layout against pages packed here field by field."""
import numpy as np
import pytest

import qsa_harness as H
from sparse_attention_decode_compress_b200 import _lib


def _pack(vals: np.ndarray, P: int, d: int, page_bytes: int) -> np.ndarray:
    """Packs values [n, P/4, d] in [-512, 508] one field at a time."""
    n, R, _ = vals.shape
    out = np.zeros((n, page_bytes), dtype=np.uint8)
    for pg in range(n):
        for row in range(R):
            for j in range(d):
                v = int(vals[pg, row, j])
                out[pg, row * d + j] = v & 255
                f = (v >> 8) + 2
                w, s, k = j // 16, (j % 16) // 4, j % 4
                out[pg, R * d + 4 * (w * R + row) + k] |= f << (2 * s)
    return out


@pytest.mark.parametrize("P,d", [(64, 128), (16, 32), (64, 64), (32, 32), (16, 128), (4, 128),
                                 (8, 32), (12, 64), (20, 128), (4, 32)])
def test_page_bytes(P, d):
    lib = _lib.load()
    R = P // 4
    assert lib.qsa_kc_page_bytes(P, d) == R * d + -(-(R * d // 4) // 16) * 16
    assert lib.qsa_kc_page_bytes(P, d) % 16 == 0


def test_page_bytes_rejects_bad_geometry():
    lib = _lib.load()
    assert lib.qsa_kc_page_bytes(6, 128) == 0   # pages hold whole micro-blocks: P % 4 == 0
    assert lib.qsa_kc_page_bytes(2, 32) == 0
    assert lib.qsa_kc_page_bytes(64, 48) == 0
    assert lib.qsa_kc_page_bytes(0, 128) == 0


@pytest.mark.parametrize("P,d", [(64, 128), (16, 32), (32, 64), (4, 128), (12, 32), (20, 64)])
def test_harness_reader_round_trip(P, d):
    lib = _lib.load()
    rng = np.random.default_rng(P * d)
    vals = rng.integers(-512, 509, size=(3, P // 4, d))
    vals[0, 0, :4] = [-512, 508, -1, 0]   # extremes and the field boundary
    vals[0, 0, 4:8] = [255, 256, -256, -257]
    pages = _pack(vals, P, d, int(lib.qsa_kc_page_bytes(P, d)))
    assert np.array_equal(H.unpack_kc_pages(pages, P, d), vals)


def test_cache_allocation_uses_the_packed_page():
    import torch
    from sparse_attention_decode_compress_b200 import QSACache
    k = torch.zeros((5, 64, 2, 128), dtype=torch.bfloat16)
    bt = torch.zeros((1, 5), dtype=torch.int32)
    c = QSACache.allocate(k, k.clone(), bt, idx_dim=128, ring_rows=1)
    assert c.kc.dtype == torch.uint8 and tuple(c.kc.shape) == (5, 16 * 128 + 16 * 32)
    k8 = torch.zeros((5, 8, 2, 128), dtype=torch.bfloat16)
    c8 = QSACache.allocate(k8, k8.clone(), bt, idx_dim=128, ring_rows=1)
    assert tuple(c8.kc.shape) == (5, 2 * 128 + 64)
    k6 = torch.zeros((5, 6, 2, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="unsupported compressed-key geometry"):
        QSACache.allocate(k6, k6.clone(), bt, idx_dim=128, ring_rows=1)
    # an int16-shaped cache is rejected before any pointer is taken
    bad = QSACache(k, k.clone(), torch.zeros((5, 4096), dtype=torch.uint8), c.ring, bt)
    with pytest.raises(ValueError, match="qsa_kc_page_bytes"):
        bad.struct()
