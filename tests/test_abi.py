"""The C-ABI library loads, exports every entry point include/qsa.h declares,
and rejects malformed host-side arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

from sparse_attention_decode_compress_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    with open(os.path.join(ROOT, "include", "qsa.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qsa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_path():
    names = _declared_functions()
    for n in ("qsa_compress_append", "qsa_index_topk", "qsa_sparse_decode", "qsa_lse_merge",
              "qsa_get_device_error"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    for name in _declared_functions():
        assert hasattr(lib, name), name
    assert set(_declared_functions()) == set(_lib.SIGNATURES)


def test_status_strings_and_version():
    lib = _lib.load()
    assert lib.qsa_abi_version() == 2
    assert lib.qsa_status_string(0) == b"QSA_OK"
    assert b"BOUNDS" in lib.qsa_status_string(3)
    assert b"unknown" in lib.qsa_status_string(99)


def test_workspace_sizes():
    lib = _lib.load()
    tick = 64 * 1024
    # header, the group maxima (one per 16 blocks), the scores
    assert lib.qsa_index_topk_workspace_bytes(128, 65536) == tick + 128 * 4096 * 4 + 128 * 65536 * 4
    assert lib.qsa_index_topk_workspace_bytes(-1, 3) == 0
    # decode: B*Hkv*nch slots of (M*D floats + M floats), nch = ceil((topk+2)/32) + S - 1
    # (room for the smallest chunks, 32 micro-blocks, a launch may pick)
    B, T, Hq, Hkv, D, K, S = 128, 1, 16, 2, 128, 512, 2
    nch = -(-(K + 2) // 32) + S - 1
    M = Hq // Hkv * T
    def al(x):
        return -(-x // 256) * 256
    want = tick + al(B * Hkv * nch * M * D * 4) + al(B * Hkv * nch * M * 4)
    assert lib.qsa_sparse_decode_workspace_bytes(B, T, Hq, Hkv, D, K, S) == want


def _cache(**kw):
    c = _lib.QsaCacheStruct()
    c.num_pages, c.page_size, c.num_kv_heads, c.head_dim, c.idx_dim = 16, 64, 2, 128, 128
    c.kv_dtype = 1
    fake = 0x10000
    c.k_cache = c.v_cache = c.kc = c.ring = c.block_table = fake
    c.ring_rows, c.max_pages_per_req = 4, 8
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("field,value", [("page_size", 6), ("page_size", 0), ("num_pages", 0),
                                         ("block_table", None)])
def test_bad_cache_rejected_on_host(field, value):
    lib = _lib.load()
    c = _cache(**{field: value})
    st = lib.qsa_compress_append(ctypes.byref(c), 1, 0x100, 0x100, 0x100, 1, None)
    assert st == 1                                   # QSA_ERR_INVALID_ARG
    st = lib.qsa_index_topk(ctypes.byref(c), 1, 0x100, 0x100, None, 16, 8, 0x100, None, 0x100,
                            1 << 20, None)
    assert st == 1


def test_bad_sizes_rejected_on_host():
    lib = _lib.load()
    c = _cache()
    assert lib.qsa_compress_append(ctypes.byref(c), 5, 0x100, 0x100, 0x100, 1, None) == 1  # B > ring
    assert lib.qsa_index_topk(ctypes.byref(c), 1, 0x100, 0x100, None, 16, 0, 0x100, None, 0x100,
                              1 << 20, None) == 1      # topk 0
    assert lib.qsa_index_topk(ctypes.byref(c), 1, 0x100, 0x100, None, 16, 8, 0x100, None, 0x100,
                              16, None) == 1           # workspace too small
    # decode: Hq not a multiple of Hkv, too many rows, unsupported dtype pairing
    assert lib.qsa_sparse_decode(ctypes.byref(c), 1, 1, 15, 0x100, 1, 0x100, 0x100, 8, 0.1, 2,
                                 0x100, 0x100, 0x100, 1 << 20, None) == 1
    assert lib.qsa_sparse_decode(ctypes.byref(c), 1, 4, 32, 0x100, 1, 0x100, 0x100, 8, 0.1, 2,
                                 0x100, 0x100, 0x100, 1 << 20, None) == 2
    assert lib.qsa_sparse_decode(ctypes.byref(c), 1, 1, 16, 0x100, 0, 0x100, 0x100, 8, 0.1, 2,
                                 0x100, 0x100, 0x100, 1 << 20, None) == 2
    assert lib.qsa_sparse_decode(ctypes.byref(c), 1, 1, 16, 0x100, 1, 0x100, 0x100, 8, 0.1, 17,
                                 0x100, 0x100, 0x100, 1 << 20, None) == 1
    assert lib.qsa_lse_merge(2, 10, 3, 0x100, 0x100, 0x100, 0x100, None) == 1
    assert lib.qsa_lse_merge(0, 10, 4, 0x100, 0x100, 0x100, 0x100, None) == 1
    # nothing to do is OK and launches nothing
    assert lib.qsa_lse_merge(2, 0, 4, None, None, None, None, None) == 0
    assert lib.qsa_index_topk(ctypes.byref(c), 0, None, None, None, 16, 8, None, None, None, 0,
                              None) == 0


def test_page_sizes_of_whole_micro_blocks_have_packed_pages():
    # any page of whole 4-token micro-blocks is a valid geometry (PR #53896
    # report, 实现拆解: the block size must be divisible by the compress
    # ratio); the calls themselves run on the GPU tests only
    lib = _lib.load()
    for P in (4, 8, 12, 20, 24, 36):
        assert lib.qsa_kc_page_bytes(P, 128) > 0
    for P in (2, 6, 10, 18):
        assert lib.qsa_kc_page_bytes(P, 128) == 0


def test_norm_indexer_rejects_bad_arguments_on_the_host():
    lib = _lib.load()
    c = _cache()
    assert lib.qsa_kcn_page_bytes(64, 128) == 16 * 128 * 2
    assert lib.qsa_kcn_page_bytes(12, 32) == 3 * 32 * 2
    assert lib.qsa_kcn_page_bytes(6, 128) == 0 and lib.qsa_kcn_page_bytes(64, 48) == 0
    # eps must be positive; pointers 16-byte aligned; B within the ring
    assert lib.qsa_compress_append_norm(ctypes.byref(c), 0x100, 0x100, None, 0.0, 1, 0x100,
                                        0x100, 0x100, 1, None) == 1
    assert lib.qsa_compress_append_norm(ctypes.byref(c), 0x108, 0x100, None, 1e-6, 1, 0x100,
                                        0x100, 0x100, 1, None) == 1
    assert lib.qsa_compress_append_norm(ctypes.byref(c), 0x100, 0x100, None, 1e-6, 5, 0x100,
                                        0x100, 0x100, 1, None) == 1
    c48 = _cache(idx_dim=48)
    assert lib.qsa_compress_append_norm(ctypes.byref(c48), 0x100, 0x100, None, 1e-6, 1, 0x100,
                                        0x100, 0x100, 1, None) == 2
    # topk out of range, workspace too small, misaligned query
    assert lib.qsa_index_topk_norm(ctypes.byref(c), 0x100, 1, 0x100, 0x100, None, 16, 0, 0x100,
                                   None, 0x100, 1 << 20, None) == 1
    assert lib.qsa_index_topk_norm(ctypes.byref(c), 0x100, 1, 0x100, 0x100, None, 16, 8, 0x100,
                                   None, 0x100, 16, None) == 1
    assert lib.qsa_index_topk_norm(ctypes.byref(c), 0x100, 1, 0x104, 0x100, None, 16, 8, 0x100,
                                   None, 0x100, 1 << 20, None) == 1
    assert lib.qsa_index_topk_norm(ctypes.byref(c), 0x100, 0, None, None, None, 16, 8, None, None,
                                   None, 0, None) == 0


def test_sparse_prefill_rejects_bad_arguments_on_the_host():
    lib = _lib.load()
    c = _cache()
    assert lib.qsa_sparse_prefill_workspace_bytes(0, 16, 16, 2, 128, 8) > 0
    assert lib.qsa_sparse_prefill_workspace_bytes(4, 0, 16, 2, 128, 8) == 0
    ok = dict(B=1, n=4, maxq=4, cu=0x100, lens=0x100, qi=0x100, kc=0x100, q=0x100, qd=1, Hq=16,
              mb=16, topk=8, sm=0.1, sel=0x100, o=0x100, lse=0x100, ws=0x100, wsb=1 << 30)

    def call(**kw):
        a = dict(ok, **kw)
        return lib.qsa_sparse_prefill(ctypes.byref(c), a["B"], a["n"], a["maxq"], a["cu"],
                                      a["lens"], a["qi"], a["kc"], a["q"], a["qd"], a["Hq"],
                                      a["mb"], a["topk"], a["sm"], a["sel"], a["o"], a["lse"],
                                      a["ws"], a["wsb"], None)
    assert call(topk=0) == 1
    assert call(mb=0) == 1
    assert call(qi=0x108) == 1            # indexer queries 16-byte aligned
    assert call(ws=0x180) == 1            # workspace 256-byte aligned
    assert call(wsb=16) == 1              # workspace too small
    assert call(Hq=15) == 1               # Hq % Hkv
    assert call(n=70000) == 2             # more query tokens than one call takes
    assert call(B=0) == 0 and call(n=0) == 0   # nothing to do
