"""The C ABI library: it loads, exports every declared symbol, and rejects bad
arguments on the host (no GPU work is enqueued by these calls)."""
import ctypes
import os
import re

import pytest

from long_context_sparse_10_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"CSA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from long_context_sparse_10_b200 import build
        build.build()
    return _lib.load()


def test_header_declares_the_five_method_calls():
    names = _declared()
    for n in ("csa_compress", "csa_indexer_topk", "csa_sparse_mqa", "hca_compress", "hca_dense_mqa"):
        assert n in names


def test_every_declared_symbol_is_exported_and_bound(lib):
    names = _declared()
    assert names, "no declarations found"
    for n in names:
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, f"{n} has no ctypes signature"
    assert set(_lib.SIGNATURES) == set(names)


def test_version_and_status_strings(lib):
    assert b"sm_100a" in lib.csa_version()
    assert lib.csa_status_string(0) == b"CSA_OK"
    assert lib.csa_status_string(3) == b"CSA_ERR_WORKSPACE"


def test_struct_layouts_match_header():
    assert ctypes.sizeof(_lib.KVCacheDesc) == 4 + 4 + 8 + 5 * 8
    assert ctypes.sizeof(_lib.WindowDesc) == 8 + 8 + 8 + 8 + 4 + 4


def test_host_side_argument_errors(lib):
    INV = _lib.CSA_ERR_INVALID_ARG
    # NULL input with real sizes
    assert lib.csa_compress(None, 1, 16, 192, 4, None, None, 0, None, None, None, None) == INV
    assert b"x is NULL" in lib.csa_last_error()
    # d not a multiple of 8
    assert lib.csa_compress(None, 1, 16, 190, 4, None, None, 0, None, None, None, None) == INV
    # split FP8 needs d == 192
    assert lib.hca_compress(None, 1, 16, 128, 128, None, None, 1, None, None, None, None) == _lib.CSA_ERR_UNSUPPORTED
    # bad m
    assert lib.csa_compress(None, 1, 16, 192, 0, None, None, 0, None, None, None, None) == INV
    # misaligned pointer
    assert lib.csa_compress(8, 1, 16, 192, 4, 16, 16, 0, 16, None, None, None) == INV
    assert b"not 16-byte aligned" in lib.csa_last_error()
    # k out of range
    assert lib.csa_indexer_topk(None, None, None, 1, 1, 10, 0, 4, 0, None, None, 0, None) == INV
    assert lib.csa_indexer_topk(None, None, None, 1, 1, 10, 0, 4, 5000, None, None, 0, None) == INV
    # H unsupported
    cd = _lib.KVCacheDesc()
    assert lib.hca_dense_mqa(16, 1, 1, 32, 0, ctypes.byref(cd), 128, None, 0.1, 16, None, None, 0, None) == INV
    # unknown cache layout
    cd.layout = 7
    assert lib.hca_dense_mqa(16, 1, 1, 64, 0, ctypes.byref(cd), 128, None, 0.1, 16, None, None, 0, None) == INV
    # a negative SM budget
    assert lib.hca_dense_mqa_budget(16, 1, 1, 64, 0, ctypes.byref(cd), 128, None, 0.1, 16, None, -1, None, 0,
                                    None) == INV
    assert b"max_sms" in lib.csa_last_error()
    # sparse attention needs idx
    cd.layout = 0
    assert lib.csa_sparse_mqa(16, 1, 1, 64, 0, ctypes.byref(cd), 4, None, 8, None, 0.1, 16, None, None, 0,
                              None) == INV
    # empty problems are no-ops
    assert lib.csa_compress(None, 0, 16, 192, 4, None, None, 0, None, None, None, None) == _lib.CSA_OK
    assert lib.csa_indexer_topk(None, None, None, 0, 5, 10, 0, 4, 8, None, None, 0, None) == _lib.CSA_OK


def test_window_must_cover_every_query(lib):
    cd = _lib.KVCacheDesc()
    wd = _lib.WindowDesc()
    wd.k = 16
    wd.pos0 = 100
    wd.rows = 50
    wd.len = 128
    # query at position 120 needs raw rows from max(0, 120-127) = 0, but the buffer starts at 100
    st = lib.hca_dense_mqa(16, 1, 1, 64, 120, ctypes.byref(cd), 128, ctypes.byref(wd), 0.1, 16, None, None, 0, None)
    assert st == _lib.CSA_ERR_INVALID_ARG
    assert b"do not cover" in lib.csa_last_error()


def test_workspace_sizes_are_monotone(lib):
    a = lib.csa_indexer_topk_workspace_size(8, 1, 262144, 2048)
    b = lib.csa_indexer_topk_workspace_size(8, 1, 131072, 2048)
    assert a > b > 0
    assert lib.csa_indexer_topk_workspace_size(0, 1, 10, 4) == 0


def test_long_row_indexer_workspace_layout(lib):
    """Decode rows (long-row path): fp32 scores (rows padded to 4 entries), the 4096-bin histograms and
    candidate counters (zeroed per call), the per-row threshold pair and per-8192-entry-chunk counts, the
    (key, index) candidate lists and the bitmaps (rows padded to 16 words), each region 256-byte aligned."""
    def up(x):
        return (x + 255) // 256 * 256

    for R, N in ((8, 262144), (64, 32768), (2, 300001), (3, 50000)):
        pitch = (N + 3) // 4 * 4
        W = ((N + 31) // 32 + 15) // 16 * 16
        nch = -(-N // 8192)
        off = up(R * pitch * 4)
        off = up(off + R * 4096 * 4 + R * 4)
        off = up(off + R * 8)
        off = up(off + R * nch * 4)
        off = up(off + R * N * 8)
        off = up(off + R * W * 4)
        assert lib.csa_indexer_topk_workspace_size(R, 1, N, 2048) == off, (R, N)


def test_attention_workspace_rule(lib):
    """H = 64 rows too few to fill the device split their keys over several
    CTAs and need merge records; H = 16, many rows, or one tile need none."""
    rec = (128 + 4) * 4
    sms = 148  # the library's SM count when no device is visible
    # decode: 8 rows x (2048 selected + 128 window) slots = 17 tiles of 128 keys
    assert lib.csa_sparse_mqa_workspace_size(8, 1, 64, 2048, 128) == 8 * 17 * 64 * rec
    # 8 rows x (8192 entries + 128 window) = 65 tiles over at most 148 // 8 = 18 splits
    tps = -(-65 // (sms // 8))
    assert lib.hca_dense_mqa_workspace_size(8, 1, 64, 8192, 128) == 8 * (-(-65 // tps)) * 64 * rec
    assert lib.csa_sparse_mqa_workspace_size(8, 1, 16, 2048, 128) == 0
    assert lib.csa_sparse_mqa_workspace_size(1, sms, 64, 2048, 128) == 0
    assert lib.csa_sparse_mqa_workspace_size(4, 1, 64, 100, 0) == 0
    assert lib.csa_sparse_mqa_workspace_size(0, 1, 64, 100, 0) == 0


def test_checked_build_exports_the_same_abi():
    # libcsa_checked.so (-DCSA_CHECKED: bounds checks on the gather rows) is a drop-in
    # replacement selected with CSA_LIBRARY; it must export exactly the declared calls too
    from long_context_sparse_10_b200 import build
    path = build.LIB_CHECKED
    if not os.path.exists(path):
        build.build(checked=True)
    checked = ctypes.CDLL(path)
    for n in _declared():
        assert hasattr(checked, n), n
    assert b"sm_100a" in ctypes.CFUNCTYPE(ctypes.c_char_p)(("csa_version", checked))()
