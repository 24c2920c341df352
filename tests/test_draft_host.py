"""Host-side rules of the MTP draft driver (no GPU): a draft step needs a
selection to reuse, and only max_draft of them reuse one."""
import pytest
import torch

from sparse_attention_decode_compress_b200 import QSACache, QSADraftDecode


def _driver(max_draft=3):
    k = torch.zeros((4, 64, 2, 128), dtype=torch.bfloat16)
    bt = torch.zeros((2, 4), dtype=torch.int32)
    cache = QSACache.allocate(k, k.clone(), bt, idx_dim=128, ring_rows=2)
    return QSADraftDecode(cache, 2, 16, 2048, 2, 64, max_draft=max_draft)


def test_draft_needs_a_selection_first():
    d = _driver()
    with pytest.raises(RuntimeError, match="select"):
        d.draft(None, None, torch.zeros((2, 2, 16, 128)), None)


def test_bad_budget_or_draft_count():
    k = torch.zeros((4, 64, 2, 128), dtype=torch.bfloat16)
    bt = torch.zeros((2, 4), dtype=torch.int32)
    cache = QSACache.allocate(k, k.clone(), bt, idx_dim=128, ring_rows=2)
    with pytest.raises(ValueError):
        QSADraftDecode(cache, 2, 16, 2050, 2, 64)
    with pytest.raises(ValueError):
        QSADraftDecode(cache, 2, 16, 2048, 2, 64, max_draft=4)


def test_buffers_cover_every_draft_step():
    d = _driver(max_draft=2)
    assert [o.shape[1] for o in d.o] == [1, 2, 3]
    assert d.tokens.shape == (2, 2048) and d.sel.shape == (2, 512)
