"""csa_indexer_topk_noalloc: the indexer top-k for callers that cannot allocate
device memory (for example a plugin whose host application owns every device
allocation, or code on a latency-critical path that must not call cudaMalloc).
It uses the library's static device scratch instead of a caller workspace, so
two calls in a row must each give exactly the indices of csa_indexer_topk
(index output: bit-exact), and oversize problems must be refused up front.

Kept in its own file, collected last, so a stop-at-first-failure run has run
every other test before it."""
import ctypes

import numpy as np
import pytest
import torch

from long_context_sparse_10_b200 import _lib

pytestmark = pytest.mark.gpu


def _case(seed, B, Tq, N):
    g = np.random.default_rng(seed)
    qI = torch.from_numpy(g.standard_normal((B, Tq, 4, 64)).astype(np.float32)).to(torch.bfloat16).cuda()
    wI = torch.from_numpy(g.random((B, Tq, 4)).astype(np.float32)).cuda()
    kI = torch.from_numpy(g.standard_normal((B, N, 64)).astype(np.float32)).to(torch.bfloat16).cuda()
    return qI, wI, kI


def _with_workspace(lib, qI, wI, kI, q_pos0, m, k, stream):
    B, Tq, N = qI.shape[0], qI.shape[1], kI.shape[1]
    idx = torch.full((B, Tq, k), -7, dtype=torch.int32, device="cuda")
    need = lib.csa_indexer_topk_workspace_size(B, Tq, N, k)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    st = lib.csa_indexer_topk(qI.data_ptr(), wI.data_ptr(), kI.data_ptr(), B, Tq, N, q_pos0, m, k, idx.data_ptr(),
                              ws.data_ptr(), ws.numel(), stream)
    assert st == 0, lib.csa_last_error()
    return idx


def _no_alloc(lib, qI, wI, kI, q_pos0, m, k, stream):
    B, Tq, N = qI.shape[0], qI.shape[1], kI.shape[1]
    idx = torch.full((B, Tq, k), -7, dtype=torch.int32, device="cuda")
    st = lib.csa_indexer_topk_noalloc(qI.data_ptr(), wI.data_ptr(), kI.data_ptr(), B, Tq, N, q_pos0, m, k,
                                      idx.data_ptr(), stream)
    assert st == 0, lib.csa_last_error()
    return idx


def test_no_alloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    lib = _lib.load()
    stream = torch.cuda.current_stream().cuda_stream
    # two different problems back to back: a long decode row set, then prefill rows
    cases = [(_case(1, 3, 1, 50000), 4 * 50000 - 1, 4, 2048),
             (_case(2, 1, 600, 150), 0, 4, 64)]
    for (qI, wI, kI), q_pos0, m, k in cases:
        ref = _with_workspace(lib, qI, wI, kI, q_pos0, m, k, stream)
        got = _no_alloc(lib, qI, wI, kI, q_pos0, m, k, stream)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
    # and the first problem again, after the scratch holds the second one's data
    (qI, wI, kI), q_pos0, m, k = cases[0]
    again = _no_alloc(lib, qI, wI, kI, q_pos0, m, k, stream)
    torch.cuda.synchronize()
    assert torch.equal(again, _with_workspace(lib, qI, wI, kI, q_pos0, m, k, stream))


def test_no_alloc_refuses_sizes_beyond_its_static_scratch():
    lib = _lib.load()
    # 64 rows x 2^20 entries needs far more than the 32 MiB static scratch
    st = lib.csa_indexer_topk_noalloc(None, None, None, 64, 1, 1 << 20, (4 << 20) - 1, 4, 2048, None, None)
    assert st == _lib.CSA_ERR_UNSUPPORTED
    assert b"static scratch" in lib.csa_last_error()
